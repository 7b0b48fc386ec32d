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
// FP8 E4M3 codes with one fp32 scale (low-precision router keys).  KF is the
// key format when known at compile time (the build kernels, which then carry
// no code, and no registers, for the other formats), or -1 for p.kfmt.
template <int N, int KF = -1>
__device__ void store_node_key(const Params& p, void* tree, int lev, int64_t seq, int g,
                               int64_t j, int ref, int lane, const float* key) {
  const int kf = KF >= 0 ? KF : p.kfmt;
  if (kf == RECSA_KEYS_FP8)
    store_key_fp8<N>(level_kcodes(p, tree, lev, seq, g) + (j * p.nref + ref) * p.kcb,
                     level_kscales(p, tree, lev, seq, g) + j * p.nref + ref, lane, key);
  else if (kf == RECSA_KEYS_NVFP4)
    store_key_nvfp4<N>(level_kcodes(p, tree, lev, seq, g) + (j * p.nref + ref) * p.kcb,
                       level_kbscales(p, tree, lev, seq, g) + (j * p.nref + ref) * (p.d / 16),
                       level_kscales(p, tree, lev, seq, g) + j * p.nref + ref, lane, key);
  else
    RowIO<float, N>::store(level_keys(p, tree, lev, seq, g) + (j * p.nref + ref) * p.d, lane,
                           key);
}

// Pool node j of level lev >= 2 for reference ref from its b children's
// stored keys (decoded when FP8) and values; KF as for store_node_key.
template <int N, int KF = -1>
__device__ void pool_parent(const Params& p, void* tree, int lev, int64_t seq, int g, int64_t j,
                            int ref, const float* rl, int lane, float* key, float* val) {
  const float* cv = level_vals(p, tree, lev - 1, seq, g) + j * p.b * p.d;
  const int kf = KF >= 0 ? KF : p.kfmt;
  if (kf == RECSA_KEYS_FP8) {
    const unsigned char* cc =
        level_kcodes(p, tree, lev - 1, seq, g) + (j * p.b * p.nref + ref) * p.kcb;
    const float* cs = level_kscales(p, tree, lev - 1, seq, g) + j * p.b * p.nref + ref;
    pool_children<float, N>(
        [&](int i, float* x) {
          load_key_fp8<N>(cc + int64_t(i) * p.nref * p.kcb, cs[int64_t(i) * p.nref], lane, x);
        },
        cv, p.b, p.d, rl, p.inv_sqrt_d, lane, key, val);
  } else if (kf == RECSA_KEYS_NVFP4) {
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

// pool_rows for bf16 leaf rows, with the same arithmetic in the same order
// (so the same bits), arranged for the HBM stream: a lane holds its channels
// of a row as packed bf16 words (half the registers of floats), the row
// stride is a compile-time constant (immediate load offsets), and the loads
// of the next 2 rows are in flight while the current 2 are pooled: few
// registers, so that many warps stream at once.
template <int N>
__device__ __forceinline__ void load_bf16_words(const __nv_bfloat16* row, int lane,
                                                unsigned* w) {
  if constexpr (N == 4) {
    const uint2 u = reinterpret_cast<const uint2*>(row)[lane];
    w[0] = u.x;
    w[1] = u.y;
  } else {
    w[0] = reinterpret_cast<const unsigned*>(row)[lane];
  }
}
__device__ __forceinline__ float2 bf16_word_to_float2(unsigned w) {
  __nv_bfloat162 h;
  memcpy(&h, &w, sizeof(h));
  return __bfloat1622float2(h);
}

template <int N>
__device__ void pool_leaf_bf16(const __nv_bfloat16* kbase, const __nv_bfloat16* vbase, int n,
                               const float* rl, float inv_sqrt_d, int lane, float* key,
                               float* val) {
  constexpr int U = 2, NW = N / 2, DD = 32 * N;   // a lane owns N of the d = 32 N channels
  unsigned ka[U][NW], va[U][NW], kb[U][NW], vb[U][NW];
  float m = -INFINITY, l = 0.f;
  float ak[N], av[N];
#pragma unroll
  for (int c = 0; c < N; ++c) ak[c] = av[c] = 0.f;
  auto issue = [&](unsigned (&kw)[U][NW], unsigned (&vw)[U][NW], int i0) {
    const __nv_bfloat16* kr = kbase + int64_t(i0) * DD;
    const __nv_bfloat16* vr = vbase + int64_t(i0) * DD;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + u < n) {
        load_bf16_words<N>(kr + u * DD, lane, kw[u]);
        load_bf16_words<N>(vr + u * DD, lane, vw[u]);
      }
  };
  auto consume = [&](const unsigned (&kw)[U][NW], const unsigned (&vw)[U][NW], int i0) {
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = 0.f;
      if (i0 + u < n) {
#pragma unroll
        for (int h = 0; h < NW; ++h) {
          const float2 f = bf16_word_to_float2(kw[u][h]);
          acc = fmaf(rl[2 * h], f.x, acc);
          acc = fmaf(rl[2 * h + 1], f.y, acc);
        }
      }
      s[u] = acc;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) s[u] = warp_sum(s[u]) * inv_sqrt_d;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < n) {
        const float mn = fmaxf(m, s[u]);
        const float sc = expf(m - mn);
        const float w = expf(s[u] - mn);
        l = l * sc + w;
#pragma unroll
        for (int h = 0; h < NW; ++h) {
          const float2 k = bf16_word_to_float2(kw[u][h]);
          const float2 v = bf16_word_to_float2(vw[u][h]);
          ak[2 * h] = fmaf(w, k.x, ak[2 * h] * sc);
          ak[2 * h + 1] = fmaf(w, k.y, ak[2 * h + 1] * sc);
          av[2 * h] += v.x;
          av[2 * h + 1] += v.y;
        }
        m = mn;
      }
    }
  };
  issue(ka, va, 0);
  for (int i0 = 0; i0 < n; i0 += 2 * U) {
    issue(kb, vb, i0 + U);
    consume(ka, va, i0);
    issue(ka, va, i0 + 2 * U);
    consume(kb, vb, i0 + U);
  }
  const float il = 1.f / l, in = 1.f / float(n);
#pragma unroll
  for (int c = 0; c < N; ++c) {
    key[c] = ak[c] * il;
    val[c] = av[c] * in;
  }
}

// Level 1: one warp per leaf block of one (sequence, KV head).  With bf16
// rows at d = 128, three CTAs per SM (at most 80 registers a thread) keep 24
// warps' row loads in flight, which the HBM stream needs (one CTA per SM, at
// the unbounded register count, reached a quarter of the bandwidth); other
// bf16 rows run two CTAs per SM.
template <typename T, int N, int KF>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? (N == 4 ? 3 : 2) : 1) leaf_kernel(Params p, const T* K, const T* V,
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
    if constexpr (sizeof(T) == 2 && N == 4)
      pool_leaf_bf16<N>(K + row0, V + row0, p.B, rl, p.inv_sqrt_d, lane, key, val);
    else
      pool_rows<T, N>(K + row0, V + row0, p.B, p.d, rl, p.inv_sqrt_d, lane, key, val);
    store_node_key<N, KF>(p, tree, 1, seq, g, j, ref, lane, key);
    if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, 1, seq, g) + j * p.d, lane, val);
  }
}

// Level lev >= 2: one warp per node, pooling b child summaries.
template <int N, int KF>
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
    pool_parent<N, KF>(p, tree, lev, seq, g, j, ref, rl, lane, key, val);
    store_node_key<N, KF>(p, tree, lev, seq, g, j, ref, lane, key);
    if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, lev, seq, g) + j * p.d, lane, val);
  }
}

// Append one token per sequence; pool the leaf and ancestors it completes.
// One CTA per sequence; warp w handles KV heads w, w + 8, ...  Compiled per
// key format, as the build kernels are.
template <typename T, int N, int KF>
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
        store_node_key<N, KF>(p, tree, 1, seq, g, j, ref, lane, key);
        if (ref == 0) RowIO<float, N>::store(level_vals(p, tree, 1, seq, g) + j * p.d, lane, val);
        int64_t idx = j;
        for (int lev = 2; lev <= p.lay.levels && (idx + 1) % p.b == 0; ++lev) {
          idx = (idx + 1) / p.b - 1;
          __syncwarp();
          pool_parent<N, KF>(p, tree, lev, seq, g, idx, ref, rl, lane, key, val);
          store_node_key<N, KF>(p, tree, lev, seq, g, idx, ref, lane, key);
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

template <typename T, int N, int KF>
cudaError_t build_format(const Params& p, const void* K, const void* V, const int64_t* len_host,
                         const float* r, int64_t r_stride, void* tree, cudaStream_t s) {
  const int warps = 8;
  for (int64_t seq = 0; seq < p.batch; ++seq) {
    int64_t n = len_host[seq] / p.B;
    if (n == 0) continue;
    dim3 grid(unsigned((n + warps - 1) / warps), p.hkv);
    leaf_kernel<T, N, KF><<<grid, warps * 32, 0, s>>>(p, reinterpret_cast<const T*>(K),
                                                  reinterpret_cast<const T*>(V), r, r_stride,
                                                  tree, seq, n);
    for (int lev = 2; lev <= p.lay.levels; ++lev) {
      n /= p.b;
      if (n == 0) break;
      dim3 g2(unsigned((n + warps - 1) / warps), p.hkv);
      parent_kernel<N, KF><<<g2, warps * 32, 0, s>>>(p, r, r_stride, tree, seq, lev, n);
    }
  }
  return cudaGetLastError();
}

template <typename T, int N>
cudaError_t build_typed(const Params& p, const void* K, const void* V, const int64_t* len_host,
                        const float* r, int64_t r_stride, void* tree, cudaStream_t s) {
  if (p.kfmt == RECSA_KEYS_FP8)
    return build_format<T, N, RECSA_KEYS_FP8>(p, K, V, len_host, r, r_stride, tree, s);
  if (p.kfmt == RECSA_KEYS_NVFP4)
    return build_format<T, N, RECSA_KEYS_NVFP4>(p, K, V, len_host, r, r_stride, tree, s);
  return build_format<T, N, RECSA_KEYS_F32>(p, K, V, len_host, r, r_stride, tree, s);
}

template <typename T, int N>
cudaError_t append_typed(const Params& p, void* K, void* V, const void* k_new, const void* v_new,
                         int64_t* len_dev, const float* r, int64_t r_stride, void* tree,
                         cudaStream_t s) {
  const dim3 grid(p.batch);
  T* Kt = static_cast<T*>(K);
  T* Vt = static_cast<T*>(V);
  const T* kn = static_cast<const T*>(k_new);
  const T* vn = static_cast<const T*>(v_new);
  if (p.kfmt == RECSA_KEYS_FP8)
    append_kernel<T, N, RECSA_KEYS_FP8><<<grid, 256, 0, s>>>(p, Kt, Vt, kn, vn, len_dev, r,
                                                             r_stride, tree);
  else if (p.kfmt == RECSA_KEYS_NVFP4)
    append_kernel<T, N, RECSA_KEYS_NVFP4><<<grid, 256, 0, s>>>(p, Kt, Vt, kn, vn, len_dev, r,
                                                               r_stride, tree);
  else
    append_kernel<T, N, RECSA_KEYS_F32><<<grid, 256, 0, s>>>(p, Kt, Vt, kn, vn, len_dev, r,
                                                             r_stride, tree);
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
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? append_typed<__nv_bfloat16, 4>(p, K, V, k_new, v_new, len_dev, r, r_stride,
                                                      tree, s)
                      : append_typed<__nv_bfloat16, 2>(p, K, V, k_new, v_new, len_dev, r, r_stride,
                                                      tree, s);
  return p.d == 128 ? append_typed<float, 4>(p, K, V, k_new, v_new, len_dev, r, r_stride, tree, s)
                    : append_typed<float, 2>(p, K, V, k_new, v_new, len_dev, r, r_stride, tree, s);
}

}  // namespace recsa
