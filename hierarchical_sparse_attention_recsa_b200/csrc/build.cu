// Tree build and append kernels, and the RoPE table.
//
// Pooling (one node from its children): weights = softmax_i(r . x_i / sqrt(d)),
// key = sum_i weight_i x_i, value = mean of the children's values
// ("Recursive Sparse Attention: Million-Token Length Extrapolation at
// Logarithmic Cost", abstract: one key and one mean-pooled value per node, one
// pooler per layer shared by all levels; "Subquadratic Attention with a
// Hierarchical Tree-Structured Indexer", Figure 3: higher levels pool the
// summaries of lower levels).  One warp pools one node with an online
// softmax, so K and V are streamed exactly once; each lane owns d/32
// contiguous channels and issues one 4..16-byte load per row.  With several
// reference queries (ZHA, Figure 3 caption: the key nodes of each are stored
// in parallel) the warp pools the node once per reference, reference j's
// parent key from reference j's child keys; the value is the same for all.
#include "recsa_internal.cuh"
#include "pool.cuh"

namespace recsa {
namespace {

// Store the pooled key of node j (level lev, reference ref): fp32 row, or
// FP8 E4M3 codes with one fp32 scale (low-precision router keys).
template <int N>
__device__ void store_node_key(const Params& p, void* tree, int lev, int64_t seq, int g,
                               int64_t j, int ref, int lane, const float* key) {
  if (p.kfmt == RECSA_KEYS_FP8)
    store_key_fp8<N>(level_kcodes(p, tree, lev, seq, g) + (j * p.nref + ref) * p.kcb,
                     level_kscales(p, tree, lev, seq, g) + j * p.nref + ref, lane, key);
  else if (p.kfmt == RECSA_KEYS_NVFP4)
    store_key_nvfp4<N>(level_kcodes(p, tree, lev, seq, g) + (j * p.nref + ref) * p.kcb,
                       level_kbscales(p, tree, lev, seq, g) + (j * p.nref + ref) * (p.d / 16),
                       level_kscales(p, tree, lev, seq, g) + j * p.nref + ref, lane, key);
  else
    RowIO<float, N>::store(level_keys(p, tree, lev, seq, g) + (j * p.nref + ref) * p.d, lane,
                           key);
}

// Pool node j of level lev >= 2 for reference ref from its b children's
// stored keys (decoded when FP8) and values.
template <int N>
__device__ void pool_parent(const Params& p, void* tree, int lev, int64_t seq, int g, int64_t j,
                            int ref, const float* rl, int lane, float* key, float* val) {
  const float* cv = level_vals(p, tree, lev - 1, seq, g) + j * p.b * p.d;
  if (p.kfmt == RECSA_KEYS_FP8) {
    const unsigned char* cc =
        level_kcodes(p, tree, lev - 1, seq, g) + (j * p.b * p.nref + ref) * p.kcb;
    const float* cs = level_kscales(p, tree, lev - 1, seq, g) + j * p.b * p.nref + ref;
    pool_children<float, N>(
        [&](int i, float* x) {
          load_key_fp8<N>(cc + int64_t(i) * p.nref * p.kcb, cs[int64_t(i) * p.nref], lane, x);
        },
        cv, p.b, p.d, rl, p.inv_sqrt_d, lane, key, val);
  } else if (p.kfmt == RECSA_KEYS_NVFP4) {
    const int nb = p.d / 16;
    const unsigned char* cc =
        level_kcodes(p, tree, lev - 1, seq, g) + (j * p.b * p.nref + ref) * p.kcb;
    const unsigned char* cb =
        level_kbscales(p, tree, lev - 1, seq, g) + (j * p.b * p.nref + ref) * nb;
    const float* cs = level_kscales(p, tree, lev - 1, seq, g) + j * p.b * p.nref + ref;
    pool_children<float, N>(
        [&](int i, float* x) {
          load_key_nvfp4<N>(cc + int64_t(i) * p.nref * p.kcb, cb + int64_t(i) * p.nref * nb,
                            cs[int64_t(i) * p.nref], lane, x);
        },
        cv, p.b, p.d, rl, p.inv_sqrt_d, lane, key, val);
  } else {
    const float* ck = level_keys(p, tree, lev - 1, seq, g) + (j * p.b * p.nref + ref) * p.d;
    pool_rows<float, N>(ck, cv, p.b, p.d, rl, p.inv_sqrt_d, lane, key, val,
                        int64_t(p.nref) * p.d);
  }
}

// Level 1: one warp per leaf block of one (sequence, KV head).
template <typename T, int N>
__global__ void __launch_bounds__(256) leaf_kernel(Params p, const T* K, const T* V,
                                                   const float* r, int64_t r_stride, void* tree,
                                                   int64_t seq, int64_t n_leaf) {
  const int lane = threadIdx.x & 31;
  const int64_t j = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int g = blockIdx.y;
  if (j >= n_leaf) return;
  const int64_t row0 = ((seq * p.hkv + g) * p.cap + j * p.B) * p.d;
  for (int ref = 0; ref < p.nref; ++ref) {
    float rl[N];
    load_r<N>(r + g * r_stride + ref * p.d, lane, rl);
    float key[N], val[N];
    pool_rows<T, N>(K + row0, V + row0, p.B, p.d, rl, p.inv_sqrt_d, lane, key, val);
    store_node_key<N>(p, tree, 1, seq, g, j, ref, lane, key);
    if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, 1, seq, g) + j * p.d, lane, val);
  }
}

// Level lev >= 2: one warp per node, pooling b child summaries.
template <int N>
__global__ void __launch_bounds__(256) parent_kernel(Params p, const float* r, int64_t r_stride,
                                                     void* tree, int64_t seq, int lev,
                                                     int64_t n_nodes) {
  const int lane = threadIdx.x & 31;
  const int64_t j = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int g = blockIdx.y;
  if (j >= n_nodes) return;
  for (int ref = 0; ref < p.nref; ++ref) {
    float rl[N];
    load_r<N>(r + g * r_stride + ref * p.d, lane, rl);
    float key[N], val[N];
    pool_parent<N>(p, tree, lev, seq, g, j, ref, rl, lane, key, val);
    store_node_key<N>(p, tree, lev, seq, g, j, ref, lane, key);
    if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, lev, seq, g) + j * p.d, lane, val);
  }
}

// Append one token per sequence; pool the leaf and ancestors it completes.
// One CTA per sequence; warp w handles KV heads w, w + 8, ...
template <typename T, int N>
__global__ void __launch_bounds__(256) append_kernel(Params p, T* K, T* V, const T* k_new,
                                                     const T* v_new, int64_t* len_dev,
                                                     const float* r, int64_t r_stride,
                                                     void* tree) {
  const int64_t seq = blockIdx.x;
  const int64_t len = len_dev[seq];
  if (len >= p.cap || len < 0) {
    if (threadIdx.x == 0) atomicOr(tree_error_word(tree), RECSA_DEVERR_APPEND_FULL);
    return;
  }
  for (int idx = threadIdx.x; idx < p.hkv * p.d; idx += blockDim.x) {
    const int g = idx / p.d, c = idx % p.d;
    const int64_t dst = ((seq * p.hkv + g) * p.cap + len) * p.d + c;
    const int64_t src = (seq * p.hkv + g) * p.d + c;
    K[dst] = k_new[src];
    V[dst] = v_new[src];
  }
  __syncthreads();
  const int64_t newlen = len + 1;
  if (newlen % p.B == 0) {
    const int lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int64_t j = newlen / p.B - 1;
    for (int g = threadIdx.x >> 5; g < p.hkv; g += nw) {
      for (int ref = 0; ref < p.nref; ++ref) {
        float rl[N];
        load_r<N>(r + g * r_stride + ref * p.d, lane, rl);
        const int64_t row0 = ((seq * p.hkv + g) * p.cap + j * p.B) * p.d;
        float key[N], val[N];
        pool_rows<T, N>(K + row0, V + row0, p.B, p.d, rl, p.inv_sqrt_d, lane, key, val);
        store_node_key<N>(p, tree, 1, seq, g, j, ref, lane, key);
        if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, 1, seq, g) + j * p.d, lane, val);
        int64_t idx = j;
        for (int lev = 2; lev <= p.lay.levels && (idx + 1) % p.b == 0; ++lev) {
          idx = (idx + 1) / p.b - 1;
          __syncwarp();
          pool_parent<N>(p, tree, lev, seq, g, idx, ref, rl, lane, key, val);
          store_node_key<N>(p, tree, lev, seq, g, idx, ref, lane, key);
          if (ref == 0)
            RowIO<float, N>::store(level_vals(p, tree, lev, seq, g) + idx * p.d, lane, val);
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) len_dev[seq] = newlen;
}

// RoPE table: row i holds (cos, sin) of i * base^(-2j/d), j < d/2, computed in
// double precision and rounded to fp32.
__global__ void rope_table_kernel(float2* table, int rows, int half, int d, double base) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= int64_t(rows) * half) return;
  const int64_t pos = idx / half;
  const int j = int(idx % half);
  const double inv = pow(base, -2.0 * double(j) / double(d));
  double s, c;
  sincos(double(pos) * inv, &s, &c);
  table[idx] = make_float2(float(c), float(s));
}

template <typename T, int N>
cudaError_t build_typed(const Params& p, const void* K, const void* V, const int64_t* len_host,
                        const float* r, int64_t r_stride, void* tree, cudaStream_t s) {
  const int warps = 8;
  for (int64_t seq = 0; seq < p.batch; ++seq) {
    int64_t n = len_host[seq] / p.B;
    if (n == 0) continue;
    dim3 grid(unsigned((n + warps - 1) / warps), p.hkv);
    leaf_kernel<T, N><<<grid, warps * 32, 0, s>>>(p, reinterpret_cast<const T*>(K),
                                                  reinterpret_cast<const T*>(V), r, r_stride,
                                                  tree, seq, n);
    for (int lev = 2; lev <= p.lay.levels; ++lev) {
      n /= p.b;
      if (n == 0) break;
      dim3 g2(unsigned((n + warps - 1) / warps), p.hkv);
      parent_kernel<N><<<g2, warps * 32, 0, s>>>(p, r, r_stride, tree, seq, lev, n);
    }
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_table(const Params& p, void* tree, double rope_base, cudaStream_t s) {
  const int half = p.d / 2;
  const int64_t n = int64_t(p.lay.rope_rows) * half;
  float2* table = reinterpret_cast<float2*>(reinterpret_cast<char*>(tree) + p.lay.rope_off);
  rope_table_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(table, p.lay.rope_rows, half, p.d,
                                                               rope_base);
  return cudaGetLastError();
}

cudaError_t launch_build(const Params& p, const void* K, const void* V, const int64_t* len_host,
                         const float* r, int64_t r_stride, void* tree, cudaStream_t s) {
  if (p.dtype == RECSA_DTYPE_BF16) {
    return p.d == 128 ? build_typed<__nv_bfloat16, 4>(p, K, V, len_host, r, r_stride, tree, s)
                      : build_typed<__nv_bfloat16, 2>(p, K, V, len_host, r, r_stride, tree, s);
  }
  return p.d == 128 ? build_typed<float, 4>(p, K, V, len_host, r, r_stride, tree, s)
                    : build_typed<float, 2>(p, K, V, len_host, r, r_stride, tree, s);
}

cudaError_t launch_append(const Params& p, void* K, void* V, const void* k_new, const void* v_new,
                          int64_t* len_dev, const float* r, int64_t r_stride, void* tree,
                          cudaStream_t s) {
  dim3 grid(p.batch);
  if (p.dtype == RECSA_DTYPE_BF16) {
    using T = __nv_bfloat16;
    if (p.d == 128)
      append_kernel<T, 4><<<grid, 256, 0, s>>>(p, (T*)K, (T*)V, (const T*)k_new, (const T*)v_new,
                                               len_dev, r, r_stride, tree);
    else
      append_kernel<T, 2><<<grid, 256, 0, s>>>(p, (T*)K, (T*)V, (const T*)k_new, (const T*)v_new,
                                               len_dev, r, r_stride, tree);
  } else {
    using T = float;
    if (p.d == 128)
      append_kernel<T, 4><<<grid, 256, 0, s>>>(p, (T*)K, (T*)V, (const T*)k_new, (const T*)v_new,
                                               len_dev, r, r_stride, tree);
    else
      append_kernel<T, 2><<<grid, 256, 0, s>>>(p, (T*)K, (T*)V, (const T*)k_new, (const T*)v_new,
                                               len_dev, r, r_stride, tree);
  }
  return cudaGetLastError();
}

}  // namespace recsa
