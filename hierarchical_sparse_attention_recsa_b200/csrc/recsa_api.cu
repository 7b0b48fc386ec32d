// C-ABI entry points: argument checks, tree layout and launches.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "recsa_internal.cuh"

using namespace recsa;

namespace recsa {
namespace {

std::mutex g_switch_mutex;
std::atomic<bool> g_switch_loaded{false};
Switches g_switches = {};

void read_switches_locked() {
  Switches sw = {};
  sw.zha_generic = getenv("RECSA_ZHA_GENERIC") != nullptr;
  sw.decode_generic = getenv("RECSA_DECODE_GENERIC") != nullptr;
  sw.prefill_generic = getenv("RECSA_PREFILL_GENERIC") != nullptr;
  sw.test_expire = getenv("RECSA_TEST_EXPIRE_WAIT") != nullptr;
  if (const char* e = getenv("RECSA_DECODE_SPLIT")) {
    int h = 0, sh = 0;
    if (sscanf(e, "%d,%d", &h, &sh) == 2 && h >= 1 && sh >= 1) {
      sw.split_hpc = h;
      sw.split_s = sh;
    }
  }
  if (const char* e = getenv("RECSA_PREFILL_PATH")) sw.prefill_path = atoi(e);
  g_switches = sw;
  g_switch_loaded.store(true, std::memory_order_release);
}

// Dynamic shared memory limits already set, per (kernel, device).
struct AttrEntry {
  const void* func;
  int dev;
  int smem;
  int nonportable;
};
std::mutex g_attr_mutex;
AttrEntry g_attr[512];
int g_attr_n = 0;

AttrEntry* attr_entry_locked(const void* func, int dev) {
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].func == func && g_attr[i].dev == dev) return &g_attr[i];
  if (g_attr_n == int(sizeof(g_attr) / sizeof(g_attr[0]))) return nullptr;
  g_attr[g_attr_n] = AttrEntry{func, dev, -1, 0};
  return &g_attr[g_attr_n++];
}

}  // namespace

const Switches& switches() {
  if (!g_switch_loaded.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_switch_mutex);
    if (!g_switch_loaded.load(std::memory_order_relaxed)) read_switches_locked();
  }
  return g_switches;
}

void reload_switches() {
  std::lock_guard<std::mutex> lock(g_switch_mutex);
  read_switches_locked();
}

cudaError_t ensure_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  AttrEntry* a = attr_entry_locked(func, dev);
  if (a && a->smem >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && a) a->smem = bytes;
  return e;
}

cudaError_t ensure_nonportable_cluster(const void* func) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  AttrEntry* a = attr_entry_locked(func, dev);
  if (a && a->nonportable) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess && a) a->nonportable = 1;
  return e;
}

}  // namespace recsa

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

recsa_status check_geometry(const recsa_geometry* g) {
  if (!g) return RECSA_ERR_NULL;
  if (g->dtype != RECSA_DTYPE_F32 && g->dtype != RECSA_DTYPE_BF16) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->head_dim != 64 && g->head_dim != 128) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->n_kv_heads < 1 || g->n_q_heads < g->n_kv_heads || g->n_q_heads % g->n_kv_heads)
    return RECSA_ERR_INVALID_GEOMETRY;
  int G = g->n_q_heads / g->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->leaf_block < 1 || g->leaf_block > 1024) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->branching < 2 || g->branching > 64) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->k < 1) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->window < 1) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->rope_enabled != 0 && g->rope_enabled != 1) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->rope_enabled && !(g->rope_base > 1.0f)) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->batch < 1 || g->capacity < 1) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->n_ref < 0 || g->n_ref > 64) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->n_ref > 1 && g->mode != RECSA_MODE_ZHA) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->key_format != RECSA_KEYS_F32 && g->key_format != RECSA_KEYS_FP8 &&
      g->key_format != RECSA_KEYS_NVFP4)
    return RECSA_ERR_INVALID_GEOMETRY;
  if (g->key_format != RECSA_KEYS_F32 && g->mode != RECSA_MODE_ZHA)
    return RECSA_ERR_INVALID_GEOMETRY;
  if (g->reserved != 0) return RECSA_ERR_INVALID_GEOMETRY;
  if (g->mode != RECSA_MODE_RECSA && g->mode != RECSA_MODE_ZHA && g->mode != RECSA_MODE_GROUP)
    return RECSA_ERR_INVALID_GEOMETRY;
  if (g->mode == RECSA_MODE_ZHA && !(g->top_p > 0.f && g->top_p <= 1.f))
    return RECSA_ERR_INVALID_GEOMETRY;
  if (g->capacity > int64_t(INT32_MAX)) return RECSA_ERR_INVALID_GEOMETRY;
  return RECSA_OK;
}

int count_levels(const recsa_geometry* g, int64_t length, int64_t* nodes) {
  int D = 0;
  int64_t span = g->leaf_block;
  while (D < kMaxLevels + 1 && length / span >= 1) {
    if (D < kMaxLevels && nodes) nodes[D] = length / span;
    ++D;
    if (span > (int64_t(1) << 50) / g->branching) break;
    span *= g->branching;
  }
  return D;
}

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

recsa_status make_layout(const recsa_geometry* g, TreeLayout* lay) {
  memset(lay, 0, sizeof(*lay));
  int D = count_levels(g, g->capacity, lay->nodes);
  if (D > kMaxLevels) return RECSA_ERR_UNSUPPORTED;
  lay->levels = D;
  const int64_t cap = g->capacity;
  const int64_t kk = std::min<int64_t>(g->k, cap);
  int64_t rows = std::max<int64_t>(g->branching * kk + g->branching,
                                   g->leaf_block * kk + int64_t(g->window) + g->leaf_block);
  rows = std::min<int64_t>(rows, cap + g->branching + 1);
  // ZHA attends at true positions: every distance up to the capacity
  if (g->mode == RECSA_MODE_ZHA) rows = std::max<int64_t>(rows, cap + 1);
  if (rows > (int64_t(1) << 24)) return RECSA_ERR_UNSUPPORTED;
  lay->rope_rows = int32_t(rows);
  int64_t off = kHeaderBytes;
  lay->rope_off = off;
  off = align_up(off + rows * (g->head_dim / 2) * 8, 256);
  for (int l = 0; l < D; ++l) {
    const int64_t rows = int64_t(g->batch) * g->n_kv_heads * lay->nodes[l];
    const int64_t bytes = rows * g->head_dim * 4;
    const int64_t nref = std::max(g->n_ref, 1);
    lay->key_off[l] = off;
    if (g->key_format == RECSA_KEYS_FP8) {   // codes, then one fp32 scale per key row
      off = align_up(off + rows * nref * g->head_dim, 256);
      lay->kscale_off[l] = off;
      off = align_up(off + rows * nref * 4, 256);
    } else if (g->key_format == RECSA_KEYS_NVFP4) {   // codes, block scales, row scales
      off = align_up(off + rows * nref * (g->head_dim / 2), 256);
      lay->kbscale_off[l] = off;
      off = align_up(off + rows * nref * (g->head_dim / 16), 256);
      lay->kscale_off[l] = off;
      off = align_up(off + rows * nref * 4, 256);
    } else {
      off = align_up(off + bytes * nref, 256);
    }
    lay->val_off[l] = off;
    off = align_up(off + bytes, 256);
  }
  lay->total = off;
  return RECSA_OK;
}

recsa_status make_params(const recsa_geometry* g, Params* p) {
  recsa_status st = check_geometry(g);
  if (st != RECSA_OK) return st;
  memset(p, 0, sizeof(*p));
  st = make_layout(g, &p->lay);
  if (st != RECSA_OK) return st;
  p->dtype = g->dtype;
  p->d = g->head_dim;
  p->hq = g->n_q_heads;
  p->hkv = g->n_kv_heads;
  p->group = g->n_q_heads / g->n_kv_heads;
  p->B = g->leaf_block;
  p->b = g->branching;
  p->k = g->k;
  p->W = g->window;
  p->rope = g->rope_enabled;
  p->mode = g->mode;
  p->top_p = g->top_p;
  p->nref = std::max(g->n_ref, 1);
  p->kfmt = g->key_format;
  p->kcb = g->key_format == RECSA_KEYS_NVFP4 ? g->head_dim / 2 : g->head_dim;
  p->batch = g->batch;
  p->cap = g->capacity;
  p->Bsh = p->bsh = -1;
  for (int sh = 0; sh < 31; ++sh) {
    if ((1 << sh) == p->B) p->Bsh = sh;
    if ((1 << sh) == p->b) p->bsh = sh;
  }
  p->inv_sqrt_d = 1.0f / sqrtf(float(g->head_dim));
  // tests of the bounded waits: the decode kernel's chain threads end with a
  // wait that nothing completes, which must expire into RECSA_DEVERR_WAIT_TIMEOUT
  p->test_expire = switches().test_expire;
  return RECSA_OK;
}

}  // namespace

// Window partials: per (sequence, query, head) an fp32 row of d + 2 (the
// window's normalised output, its max and its sum).
size_t recsa::prefill_workspace_need(const Params& p, int32_t n_q) {
  return size_t(p.batch) * size_t(n_q) * size_t(p.hq) * size_t(p.d + 2) * sizeof(float);
}

namespace {

recsa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return RECSA_OK;
  fprintf(stderr, "recsa: CUDA error: %s\n", cudaGetErrorString(e));
  return RECSA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* recsa_status_string(recsa_status s) {
  switch (s) {
    case RECSA_OK: return "ok";
    case RECSA_ERR_INVALID_GEOMETRY: return "invalid geometry";
    case RECSA_ERR_NULL: return "null pointer";
    case RECSA_ERR_MISALIGNED: return "misaligned pointer";
    case RECSA_ERR_CAPACITY: return "length or query range exceeds capacity";
    case RECSA_ERR_UNSUPPORTED: return "geometry outside kernel limits";
    case RECSA_ERR_CUDA: return "CUDA error";
    case RECSA_ERR_DEVICE: return "device error flag set";
  }
  return "unknown status";
}

recsa_status recsa_validate(const recsa_geometry* geom) {
  Params p;
  return make_params(geom, &p);
}

recsa_status recsa_num_levels(const recsa_geometry* geom, int64_t length, int32_t* levels) {
  recsa_status st = check_geometry(geom);
  if (st != RECSA_OK) return st;
  if (!levels) return RECSA_ERR_NULL;
  if (length < 0) return RECSA_ERR_CAPACITY;
  *levels = count_levels(geom, length, nullptr);
  return RECSA_OK;
}

recsa_status recsa_tree_bytes(const recsa_geometry* geom, size_t* bytes) {
  if (!bytes) return RECSA_ERR_NULL;
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  *bytes = size_t(p.lay.total);
  return RECSA_OK;
}

recsa_status recsa_trace_ints(const recsa_geometry* geom, int32_t* ints) {
  if (!ints) return RECSA_ERR_NULL;
  recsa_status st = check_geometry(geom);
  if (st != RECSA_OK) return st;
  if (geom->k > RECSA_TRACE_MAX_K) return RECSA_ERR_UNSUPPORTED;
  *ints = kTraceHead + kMaxLevels * geom->k;
  return RECSA_OK;
}

recsa_status recsa_build(const recsa_geometry* geom, const void* K, const void* V,
                         const int64_t* len_host, const float* pooler_r,
                         int64_t pooler_head_stride, void* tree, void* stream) {
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (!K || !V || !len_host || !pooler_r || !tree) return RECSA_ERR_NULL;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(tree, 256) || !aligned(pooler_r, 4))
    return RECSA_ERR_MISALIGNED;
  if (pooler_head_stride < 0) return RECSA_ERR_INVALID_GEOMETRY;
  for (int s = 0; s < geom->batch; ++s)
    if (len_host[s] < 0 || len_host[s] > geom->capacity) return RECSA_ERR_CAPACITY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = cuda_status(cudaMemsetAsync(tree, 0, kHeaderBytes, s));
  if (st != RECSA_OK) return st;
  st = cuda_status(launch_rope_table(p, tree, double(geom->rope_base), s));
  if (st != RECSA_OK) return st;
  return cuda_status(launch_build(p, K, V, len_host, pooler_r, pooler_head_stride, tree, s));
}

recsa_status recsa_append(const recsa_geometry* geom, void* K, void* V, const void* k_new,
                          const void* v_new, int64_t* len_dev, const float* pooler_r,
                          int64_t pooler_head_stride, void* tree, void* stream) {
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (!K || !V || !k_new || !v_new || !len_dev || !pooler_r || !tree) return RECSA_ERR_NULL;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(tree, 256) || !aligned(len_dev, 8) || !aligned(pooler_r, 4))
    return RECSA_ERR_MISALIGNED;
  if (pooler_head_stride < 0) return RECSA_ERR_INVALID_GEOMETRY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(launch_append(p, K, V, k_new, v_new, len_dev, pooler_r, pooler_head_stride,
                                   tree, s));
}

static recsa_status attend_common(const recsa_geometry* geom, const void* Q, const void* K,
                                  const void* V, const void* tree, const int64_t* len_dev,
                                  int64_t q_start, int32_t n_q, int decode, void* O,
                                  int32_t* trace, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (!Q || !K || !V || !tree || !O || (decode && !len_dev)) return RECSA_ERR_NULL;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(tree, 256) || (trace && !aligned(trace, 4)) || (decode && !aligned(len_dev, 8)) ||
      (workspace && !aligned(workspace, 16)))
    return RECSA_ERR_MISALIGNED;
  if (n_q < 0) return RECSA_ERR_CAPACITY;
  if (!decode && (q_start < 0 || q_start + n_q > geom->capacity)) return RECSA_ERR_CAPACITY;
  if (trace && geom->k > RECSA_TRACE_MAX_K) return RECSA_ERR_UNSUPPORTED;
  if (workspace && workspace_bytes < prefill_workspace_need(p, n_q)) return RECSA_ERR_CAPACITY;
  if (n_q == 0) return RECSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorNotSupported;
  if (p.mode == RECSA_MODE_ZHA) {
    if (!switches().zha_generic) {
      // prefill: the window (true-position RoPE there too) on tensor cores first
      const void* wpart = nullptr;
      if (!decode && workspace) {
        e = launch_prefill_window(p, Q, K, V, tree, q_start, n_q, workspace, s);
        if (e == cudaSuccess) wpart = workspace;
        else if (e != cudaErrorNotSupported) return cuda_status(e);
        else cudaGetLastError();
      }
      e = launch_zha(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O, trace, wpart, s);
    }
  } else if (decode && !switches().decode_generic) {
    e = launch_decode_cluster(p, Q, K, V, tree, len_dev, n_q, O, trace, s);
  } else if (!decode && !switches().prefill_generic) {
    const void* wpart = nullptr;
    // RECSA_PREFILL_PATH: 0 automatic, 1 window + traversal kernels only (the
    // kept leaves attended by the traversal), 2 the tensor-core leaf path with
    // the warp-per-query-head traversal, 3 the tensor-core leaf path with the
    // tree levels as parent-node tiles (the automatic choice when possible)
    const int path = switches().prefill_path;
    if (workspace && path != 1 && prefill_tc_supported(p) &&
        workspace_bytes >= prefill_tc_workspace_need(p, n_q)) {
      e = launch_prefill_tc(p, Q, K, V, tree, q_start, n_q, O, trace, workspace, s);
      if (e != cudaErrorNotSupported) return cuda_status(e);
      cudaGetLastError();
    }
    if (workspace) {
      e = launch_prefill_window(p, Q, K, V, tree, q_start, n_q, workspace, s);
      if (e == cudaSuccess) wpart = workspace;
      else if (e != cudaErrorNotSupported) return cuda_status(e);
      else cudaGetLastError();
    }
    e = launch_prefill_warp(p, Q, K, V, tree, q_start, n_q, O, trace, wpart, s);
  }
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_attend(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O, trace, s);
  }
  if (e == cudaErrorInvalidConfiguration || e == cudaErrorInvalidValue) {
    cudaGetLastError();
    return RECSA_ERR_UNSUPPORTED;
  }
  return cuda_status(e);
}

recsa_status recsa_decode(const recsa_geometry* geom, const void* Q, const void* K,
                          const void* V, const void* tree, const int64_t* len_dev,
                          int32_t n_q, void* O, int32_t* trace, void* stream) {
  return attend_common(geom, Q, K, V, tree, len_dev, 0, n_q, 1, O, trace, nullptr, 0, stream);
}

recsa_status recsa_decode_step(const recsa_geometry* geom, const void* Q, void* K, void* V,
                               const void* k_new, const void* v_new, int64_t* len_dev,
                               const float* pooler_r, int64_t pooler_head_stride, void* tree,
                               int32_t n_q, void* O, int32_t* trace, void* stream) {
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (!Q || !K || !V || !k_new || !v_new || !len_dev || !pooler_r || !tree || !O)
    return RECSA_ERR_NULL;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(k_new, 16) ||
      !aligned(v_new, 16) || !aligned(O, 16) || !aligned(tree, 256) || !aligned(len_dev, 8) ||
      !aligned(pooler_r, 4) || (trace && !aligned(trace, 4)))
    return RECSA_ERR_MISALIGNED;
  if (pooler_head_stride < 0) return RECSA_ERR_INVALID_GEOMETRY;
  if (n_q < 1) return RECSA_ERR_CAPACITY;
  if (trace && geom->k > RECSA_TRACE_MAX_K) return RECSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorNotSupported;
  if (!switches().decode_generic)
    e = launch_decode_step(p, Q, K, V, k_new, v_new, len_dev, pooler_r, pooler_head_stride,
                           tree, n_q, O, trace, s);
  if (e == cudaErrorNotSupported) {
    // outside the fused kernel's limits: the same step as two launches
    cudaGetLastError();
    e = launch_append(p, K, V, k_new, v_new, len_dev, pooler_r, pooler_head_stride, tree, s);
    if (e == cudaSuccess)
      return attend_common(geom, Q, K, V, tree, len_dev, 0, n_q, 1, O, trace, nullptr, 0,
                           stream);
  }
  if (e == cudaErrorInvalidConfiguration || e == cudaErrorInvalidValue) {
    cudaGetLastError();
    return RECSA_ERR_UNSUPPORTED;
  }
  return cuda_status(e);
}

recsa_status recsa_prefill_static(const recsa_geometry* geom, const void* Q, const void* K,
                                  const void* V, const void* tree, int64_t q_start, int32_t n_q,
                                  void* O, int32_t* trace, void* stream) {
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (!Q || !K || !V || !tree || !O) return RECSA_ERR_NULL;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(tree, 256) || (trace && !aligned(trace, 4)))
    return RECSA_ERR_MISALIGNED;
  if (n_q < 0 || q_start < 0 || q_start + n_q > geom->capacity) return RECSA_ERR_CAPACITY;
  // the fixed scratch holds the window partials of the RecSA path (ZHA uses none)
  if (p.mode == RECSA_MODE_RECSA && prefill_workspace_need(p, n_q) > prefill_static_bytes()) {
    fprintf(stderr,
            "recsa_prefill_static: %zu bytes of window partials (batch * n_q * n_q_heads * "
            "(head_dim + 2) * 4) exceed the fixed scratch of %zu bytes; split the call into "
            "smaller query ranges\n",
            prefill_workspace_need(p, n_q), prefill_static_bytes());
    return RECSA_ERR_CAPACITY;
  }
  if (trace && geom->k > RECSA_TRACE_MAX_K) return RECSA_ERR_UNSUPPORTED;
  if (n_q == 0) return RECSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorNotSupported;
  if (p.mode == RECSA_MODE_ZHA) {
    if (!switches().zha_generic)
      e = launch_zha(p, Q, K, V, tree, nullptr, q_start, n_q, 0, O, trace, nullptr, s);
  } else {
    e = launch_prefill_static(p, Q, K, V, tree, q_start, n_q, O, trace, s);
  }
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_attend(p, Q, K, V, tree, nullptr, q_start, n_q, 0, O, trace, s);
  }
  if (e == cudaErrorInvalidConfiguration || e == cudaErrorInvalidValue) {
    cudaGetLastError();
    return RECSA_ERR_UNSUPPORTED;
  }
  return cuda_status(e);
}

recsa_status recsa_prefill_workspace_bytes(const recsa_geometry* geom, int32_t n_q,
                                           size_t* bytes) {
  if (!bytes) return RECSA_ERR_NULL;
  Params p;
  recsa_status st = make_params(geom, &p);
  if (st != RECSA_OK) return st;
  if (n_q < 0) return RECSA_ERR_CAPACITY;
  *bytes = prefill_workspace_need(p, n_q);
  // the tensor-core kept-leaf path keeps more intermediates: report its size
  // where the geometry allows it (a smaller workspace selects the window path)
  if (prefill_tc_supported(p)) *bytes = std::max(*bytes, prefill_tc_workspace_need(p, n_q));
  return RECSA_OK;
}

recsa_status recsa_prefill(const recsa_geometry* geom, const void* Q, const void* K,
                           const void* V, const void* tree, int64_t q_start, int32_t n_q,
                           void* O, int32_t* trace, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return attend_common(geom, Q, K, V, tree, nullptr, q_start, n_q, 0, O, trace, workspace,
                       workspace_bytes, stream);
}

void recsa_reload_switches(void) { reload_switches(); }

recsa_status recsa_tree_error(const recsa_geometry* geom, void* tree, int32_t clear,
                              uint32_t* flags, void* stream) {
  recsa_status st = check_geometry(geom);
  if (st != RECSA_OK) return st;
  if (!tree || !flags) return RECSA_ERR_NULL;
  if (!aligned(tree, 256)) return RECSA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  st = cuda_status(cudaMemcpyAsync(&host, tree, sizeof(host), cudaMemcpyDeviceToHost, s));
  if (st != RECSA_OK) return st;
  if (clear) {
    st = cuda_status(cudaMemsetAsync(tree, 0, sizeof(uint32_t), s));
    if (st != RECSA_OK) return st;
  }
  st = cuda_status(cudaStreamSynchronize(s));
  if (st != RECSA_OK) return st;
  *flags = host;
  return RECSA_OK;
}

}  // extern "C"
