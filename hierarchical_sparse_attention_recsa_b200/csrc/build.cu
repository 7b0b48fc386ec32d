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
#include "tc05.cuh"

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

// Level 1 with R >= 4 reference queries (bf16 rows, d = 128), on the tensor
// cores in one pass over K and V: a CTA takes 128 consecutive tokens (128 / B
// leaves) of one (sequence, KV head) and computes
//   S = K r^T             [128 tokens x R]   (the pooler scores of every reference),
//   W = softmax over each leaf's B tokens of S / sqrt(d)   (registers, fp32),
//   key_l^T = K_l^T W_l   [d x R] per leaf l (the pooled keys of every reference),
// as tcgen05 TF32 MMAs into TMEM.  K (bf16) is exact in TF32; r and W are fp32
// and enter as the sum of their high and low TF32 parts (two MMAs each), so
// both products keep fp32 accuracy ("ZHA", Figure 3 caption: the key nodes of
// every reference query are stored in parallel; the scores and the pooling
// are a [B x d] x [d x R] and an [R x B] x [B x d] product per leaf).  The
// value (the mean of the leaf's values, the same for every reference) is
// summed on CUDA cores in the same token order as the one-reference kernel.
constexpr int kMrThreads = 256;
constexpr unsigned long long kMrWaitNs = 200000000ull;

template <int BL, int NR>
struct MrSmem {
  static constexpr int LPT = 128 / BL;                     // leaves per tile
  static constexpr int kA = 0;                             // K [128 tok][128 d]
  static constexpr int kA2 = kA + 128 * 128 * 4;           // K^T per leaf [128 d][BL tok]
  static constexpr int kB1 = kA2 + 128 * 128 * 4;          // r hi, lo [NR][128 d]
  static constexpr int kB1n = NR * 128 * 4;
  static constexpr int kB2 = kB1 + 2 * kB1n;               // W hi, lo per leaf [NR][BL tok]
  static constexpr int kB2n = NR * BL * 4;
  static_assert(2 * LPT * kB2n >= 16 * 128 * 4, "value partials use the W operand's bytes");
  static constexpr int kS = kB2 + 2 * LPT * kB2n;          // S [NR][128 tok] fp32
  static constexpr int kBar = kS + 128 * NR * 4;
  static constexpr int kTotal = kBar + 32;
  static constexpr int kPk = kA;       // pooled keys [LPT][NR][128] over the operands (after MMA 2)
  static constexpr int kCols = NR * (1 + LPT) <= 32 ? 32 : NR * (1 + LPT) <= 64 ? 64
                               : NR * (1 + LPT) <= 128 ? 128 : NR * (1 + LPT) <= 256 ? 256 : 512;
  static_assert(kTotal <= 227 * 1024, "multi-reference tile does not fit");
  static_assert(LPT * NR * 128 * 4 <= kBar, "pooled keys must fit over the operands");
};

__device__ __forceinline__ int kmj(int R, int r, int k) { return (k >> 2) * 16 * R + r * 16 + (k & 3) * 4; }

__device__ __forceinline__ void st_split4(unsigned char* dst, int lo_off, float a, float b,
                                          float c, float d) {
  const float ha = tc05::to_tf32(a), hb = tc05::to_tf32(b), hc = tc05::to_tf32(c),
              hd = tc05::to_tf32(d);
  *reinterpret_cast<float4*>(dst) = make_float4(ha, hb, hc, hd);
  *reinterpret_cast<float4*>(dst + lo_off) =
      make_float4(tc05::to_tf32(a - ha), tc05::to_tf32(b - hb), tc05::to_tf32(c - hc),
                  tc05::to_tf32(d - hd));
}

template <int BL, int NR, int KF>
__global__ void __launch_bounds__(kMrThreads, 1)
leaf_multiref_tc_kernel(Params p, const __nv_bfloat16* K, const __nv_bfloat16* V,
                        const float* r, int64_t r_stride, void* tree, int64_t seq,
                        int64_t n_leaf) {
  using L = MrSmem<BL, NR>;
  constexpr int LPT = L::LPT, D = 128;
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kBar + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  const int64_t j0 = int64_t(blockIdx.x) * LPT;             // first leaf of the tile
  const int nl = int(n_leaf - j0 < LPT ? n_leaf - j0 : LPT);  // leaves present
  const int ntok = nl * BL;
  const int R = p.nref;
  if (warp == 0) {
    tc05::tmem_alloc(tslot, L::kCols);
    tc05::tmem_relinquish();
  }
  if (tid == 0) {
    tc05::mbar_init(&bar[0], 1);
    tc05::mbar_init(&bar[1], 1);
    tc05::mbar_fence_init();
  }
  const __nv_bfloat16* kb = K + ((seq * p.hkv + g) * p.cap + j0 * BL) * D;
  const __nv_bfloat16* vb = V + ((seq * p.hkv + g) * p.cap + j0 * BL) * D;
  // K tile ([token][d] for the scores) and, from the same registers, every
  // leaf's K^T ([d][token] for the pooling); tokens past the leaves are zero
  for (int task = tid; task < 128 * (D / 8); task += kMrThreads) {
    const int t = task % 128, c = task / 128;
    float x[8];
    if (t < ntok) {
      const uint4 u = *reinterpret_cast<const uint4*>(kb + int64_t(t) * D + 8 * c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    *reinterpret_cast<float4*>(sm + L::kA + kmj(128, t, 8 * c)) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(sm + L::kA + kmj(128, t, 8 * c + 4)) = make_float4(x[4], x[5], x[6], x[7]);
    unsigned char* kt = sm + L::kA2 + (t / BL) * (D * BL * 4);
#pragma unroll
    for (int e = 0; e < 8; ++e) *reinterpret_cast<float*>(kt + kmj(D, 8 * c + e, t % BL)) = x[e];
  }
  // values: every thread sums 8 consecutive tokens of 8 channels (16-byte
  // loads, all issued at once); the groups are added in token order below
  float* vpart = reinterpret_cast<float*>(sm + L::kB2);    // [128 / 8 groups][128 d]
  for (int task = tid; task < (128 / 8) * (D / 8); task += kMrThreads) {
    const int tg = task % 16, c = task / 16;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    uint4 u[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int t = 8 * tg + q;
      u[q] = t < ntok ? *reinterpret_cast<const uint4*>(vb + int64_t(t) * D + 8 * c)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) vpart[tg * D + 8 * c + e] = acc[e];
  }
  __syncthreads();
  for (int task = tid; task < nl * D; task += kMrThreads) {
    const int leaf = task / D, n = task % D;
    float acc = 0.f;
    for (int q = 0; q < BL / 8; ++q) acc += vpart[(leaf * (BL / 8) + q) * D + n];
    level_vals(p, tree, 1, seq, g)[(j0 + leaf) * D + n] = acc * (1.f / float(BL));
  }
  __syncthreads();   // vpart's bytes are the W operand below
  // r of every reference query (rows >= R are zero), split into TF32 high and low parts
  for (int task = tid; task < NR * (D / 4); task += kMrThreads) {
    const int ref = task % NR, c = task / NR;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ref < R) x = *reinterpret_cast<const float4*>(r + g * r_stride + int64_t(ref) * D + 4 * c);
    st_split4(sm + L::kB1 + kmj(NR, ref, 4 * c), L::kB1n, x.x, x.y, x.z, x.w);
  }
  tc05::fence_smem_to_async();
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t aA = tc05::smem_u32(sm + L::kA), aA2 = tc05::smem_u32(sm + L::kA2);
  const uint32_t aB1 = tc05::smem_u32(sm + L::kB1), aB2 = tc05::smem_u32(sm + L::kB2);
  constexpr uint32_t id1 = tc05::idesc(tc05::kFmtTF32, 128, NR);
  if (tid == 0) {
#pragma unroll
    for (int kk = 0; kk < D / 8; ++kk) {
      const uint32_t a = aA + kk * 32 * 128, b = aB1 + kk * 32 * NR;
      tc05::mma_tf32(tmem, tc05::desc_kmajor(a, 16 * 128, 128),
                     tc05::desc_kmajor(b, 16 * NR, 128), id1, kk > 0);
      tc05::mma_tf32(tmem, tc05::desc_kmajor(a, 16 * 128, 128),
                     tc05::desc_kmajor(b + L::kB1n, 16 * NR, 128), id1, 1);
    }
    tc05::mma_commit(&bar[0]);
  }
  bool ok = __syncthreads_and(tid != 0 || tc05::mbar_wait_bounded(&bar[0], 0, kMrWaitNs));
  tc05::fence_after_sync();
  float* Ssm = reinterpret_cast<float*>(sm + L::kS);   // [NR][128 tokens]
  if (warp < 4 && ok) {
    float sv[NR];
#pragma unroll
    for (int c = 0; c < NR / 16; ++c)
      tc05::tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + 16 * c, sv + 16 * c);
    tc05::tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < NR; ++c) Ssm[c * 128 + tid] = sv[c] * p.inv_sqrt_d;
  }
  __syncthreads();
  // softmax over each leaf's tokens: one warp per (leaf, reference) column,
  // lanes over the tokens
  for (int col = warp; col < LPT * NR; col += kMrThreads / 32) {
    const int leaf = col / NR, ref = col % NR;
    const float* s = Ssm + ref * 128 + leaf * BL;
    constexpr int PER = BL >= 32 ? BL / 32 : 1;
    float x[PER];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int t = lane + 32 * e;
      x[e] = t < BL ? s[t] : -INFINITY;
      m = fmaxf(m, x[e]);
    }
    m = warp_max(m);
    float l = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      x[e] = lane + 32 * e < BL ? expf(x[e] - m) : 0.f;
      l += x[e];
    }
    const float il = 1.f / warp_sum(l);
    unsigned char* wb = sm + L::kB2 + leaf * 2 * L::kB2n;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int t = lane + 32 * e;
      if (t < BL) {
        const float w = x[e] * il, hi = tc05::to_tf32(w);
        *reinterpret_cast<float*>(wb + kmj(NR, ref, t)) = hi;
        *reinterpret_cast<float*>(wb + L::kB2n + kmj(NR, ref, t)) = tc05::to_tf32(w - hi);
      }
    }
  }
  tc05::fence_smem_to_async();
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  if (tid == 0 && ok) {
    for (int leaf = 0; leaf < LPT; ++leaf) {
      const uint32_t dcol = tmem + NR * (1 + leaf);
#pragma unroll
      for (int kk = 0; kk < BL / 8; ++kk) {
        const uint32_t a = aA2 + leaf * (D * BL * 4) + kk * 32 * D;
        const uint32_t b = aB2 + leaf * 2 * L::kB2n + kk * 32 * NR;
        tc05::mma_tf32(dcol, tc05::desc_kmajor(a, 16 * D, 128),
                       tc05::desc_kmajor(b, 16 * NR, 128), id1, kk > 0);
        tc05::mma_tf32(dcol, tc05::desc_kmajor(a, 16 * D, 128),
                       tc05::desc_kmajor(b + L::kB2n, 16 * NR, 128), id1, 1);
      }
    }
    tc05::mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(tid != 0 || !ok || tc05::mbar_wait_bounded(&bar[1], 0, kMrWaitNs)) && ok;
  tc05::fence_after_sync();
  // pooled keys: thread t of warps 0-3 holds dimension t of every (leaf, reference)
  float* Pk = reinterpret_cast<float*>(sm + L::kPk);
  if (warp < 4 && ok) {
    for (int leaf = 0; leaf < LPT; ++leaf) {
#pragma unroll
      for (int c = 0; c < NR / 16; ++c) {
        float kv[16];
        tc05::tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + NR * (1 + leaf) + 16 * c, kv);
        tc05::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) Pk[(leaf * NR + 16 * c + e) * D + tid] = kv[e];
      }
    }
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  if (ok) {
    // key rows (fp32, FP8 or NVFP4 storage, as the one-reference kernel stores them)
    for (int row = warp; row < nl * R; row += kMrThreads / 32) {
      const int leaf = row / R, ref = row % R;
      float key[4];
      RowIO<float, 4>::load(Pk + (leaf * NR + ref) * D, lane, key);
      store_node_key<4, KF>(p, tree, 1, seq, g, j0 + leaf, ref, lane, key);
    }
  } else if (tid == 0) {
    atomicOr(tree_error_word(tree), RECSA_DEVERR_WAIT_TIMEOUT);
    tc05::mbar_wait_bounded(&bar[0], 0, kMrWaitNs);
    tc05::mbar_wait_bounded(&bar[1], 0, kMrWaitNs);
  }
  __syncthreads();
  if (warp == 0) tc05::tmem_dealloc(tmem, L::kCols);
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

template <int BL, int NR, int KF>
cudaError_t launch_multiref_tc(const Params& p, const void* K, const void* V, const float* r,
                               int64_t r_stride, void* tree, int64_t seq, int64_t n,
                               cudaStream_t s) {
  using L = MrSmem<BL, NR>;
  auto kern = leaf_multiref_tc_kernel<BL, NR, KF>;
  cudaError_t e = ensure_smem(kern, L::kTotal);
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned((n + L::LPT - 1) / L::LPT), p.hkv);
  kern<<<grid, kMrThreads, L::kTotal, s>>>(p, reinterpret_cast<const __nv_bfloat16*>(K),
                                           reinterpret_cast<const __nv_bfloat16*>(V), r,
                                           r_stride, tree, seq, n);
  return cudaGetLastError();
}

// The tensor-core level-1 kernel for R >= 4 reference queries (up to 32),
// bf16 rows of d = 128 and B in {16, 32, 64}; cudaErrorNotSupported otherwise.
template <int KF>
cudaError_t leaf_multiref_dispatch(const Params& p, const void* K, const void* V, const float* r,
                                   int64_t r_stride, void* tree, int64_t seq, int64_t n,
                                   cudaStream_t s) {
  if (p.dtype != RECSA_DTYPE_BF16 || p.d != 128 || p.nref < 4 || p.nref > 32 ||
      switches().prefill_path == 1)
    return cudaErrorNotSupported;
  const bool wide = p.nref > 16;
#define RECSA_MR_CASE(BLV)                                                                  \
  if (p.B == BLV)                                                                           \
    return wide ? launch_multiref_tc<BLV, 32, KF>(p, K, V, r, r_stride, tree, seq, n, s)     \
                : launch_multiref_tc<BLV, 16, KF>(p, K, V, r, r_stride, tree, seq, n, s);
  RECSA_MR_CASE(16)
  RECSA_MR_CASE(32)
  RECSA_MR_CASE(64)
#undef RECSA_MR_CASE
  return cudaErrorNotSupported;
}

template <typename T, int N, int KF>
cudaError_t build_format(const Params& p, const void* K, const void* V, const int64_t* len_host,
                         const float* r, int64_t r_stride, void* tree, cudaStream_t s) {
  const int warps = 8;
  for (int64_t seq = 0; seq < p.batch; ++seq) {
    int64_t n = len_host[seq] / p.B;
    if (n == 0) continue;
    cudaError_t e = leaf_multiref_dispatch<KF>(p, K, V, r, r_stride, tree, seq, n, s);
    if (e == cudaErrorNotSupported) {
      cudaGetLastError();
      dim3 grid(unsigned((n + warps - 1) / warps), p.hkv);
      leaf_kernel<T, N, KF><<<grid, warps * 32, 0, s>>>(p, reinterpret_cast<const T*>(K),
                                                    reinterpret_cast<const T*>(V), r, r_stride,
                                                    tree, seq, n);
    } else if (e != cudaSuccess) {
      return e;
    }
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
