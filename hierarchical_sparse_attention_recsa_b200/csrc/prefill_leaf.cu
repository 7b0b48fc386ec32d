// Kept-leaf attention of a prefill on the tensor cores (tcgen05), regrouped
// by leaf.
//
// In a prefill every (query, head) keeps up to k leaf blocks, and they differ
// from query to query, so per query the kept leaves are a gather with no
// reuse.  Across a whole chunk of queries, though, each leaf is kept by many
// (query head, slot) pairs: 65536 queries x 32 heads x 8 slots over 8192
// leaves of 8 KV heads at 524K is about 256 pairs per leaf.  Grouping the
// pairs by leaf turns the gather into dense tiles: one leaf's B keys meet up to
// 128 pairs' queries in one [128 x d] x [d x B] product, and its values in one
// [128 x B] x [B x d] product.
//
// Candidate-local RoPE ("Recursive Sparse Attention: Million-Token Length
// Extrapolation at Logarithmic Cost", abstract) makes this possible: token j
// of the leaf in slot s of a query sits at index s B + j among its exact
// entries and the query at n0 - 1, so its logit is
//   < R(n0 - 1) q, R(s B + j) k_j > = < R(n0 - 1 - s B) q, R(j) k_j >:
// the key side is rotated by its offset in the leaf alone (the same for every
// pair) and the query side once per pair.
//
// Steps of a prefill call with this path (launch_prefill_tc):
//   1. window_mma_kernel: the exact window's partial softmax per query head;
//   2. prefill_warp_kernel: the traversal; it merges the window partial with
//      the unselected summaries into one partial (in place), lists the kept
//      leaves and counts the pairs of every leaf (atomics give each pair its
//      position in its leaf's list);
//   3. scan_kernel: exclusive prefix sum of the per-leaf counts;
//   4. scatter_kernel: the (query head, slot, query rotation) pairs, grouped by leaf;
//   5. leaf_tc_kernel: per leaf, tiles of 128 pairs on tcgen05 (TF32 operands,
//      fp32 accumulation in TMEM), one partial softmax per pair;
//   6. merge_kernel: per query head, the traversal's partial and its kept
//      leaves' partials into O.
#include <type_traits>

#include "recsa_internal.cuh"
#include "tc05.cuh"

namespace recsa {
namespace {

constexpr int kLThreads = 128;
constexpr int kTile = 64;                    // pairs per tile (MMA rows, M = 64)
constexpr unsigned long long kLeafWaitNs = 200000000ull;   // 200 ms per MMA wait

struct LeafPaths {
  float* part;       // [rows][d + 2]: window + summaries partial per query head
  float* lpart;      // [rows * kmax][d]: normalised output per (query head, slot)
  float2* lml;       // [rows * kmax]: its (max, sum)
  int2* kept;        // [rows * kmax]: {leaf bucket, position in the bucket}
  int* nkept;        // [rows]
  int* counts;       // [buckets]
  int* offsets;      // [buckets]
  int2* pairs;       // [rows * kmax]: {query-head row, slot << 24 | query rotation}
  void* tree_ws;     // the tree levels' workspace (prefill_tree.cu), or null
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int kmax_of(const Params& p) {
  const int64_t n1 = p.lay.levels > 0 ? p.lay.nodes[0] : 0;
  int64_t k = p.k < n1 ? p.k : n1;
  return int(k < 1 ? 1 : k);
}

int64_t buckets_of(const Params& p) {
  return int64_t(p.batch) * p.hkv * (p.lay.levels > 0 ? p.lay.nodes[0] : 1);
}

LeafPaths carve(const Params& p, int32_t n_q, void* ws, size_t* total) {
  const size_t rows = size_t(p.batch) * n_q * p.hq;
  const int kmax = kmax_of(p);
  const size_t nb = size_t(buckets_of(p));
  size_t off[10];
  off[0] = 0;                                                  // part
  off[1] = align256(off[0] + rows * (p.d + 2) * 4);            // lpart
  off[2] = align256(off[1] + rows * kmax * p.d * 4);           // lml
  off[3] = align256(off[2] + rows * kmax * 8);                 // kept
  off[4] = align256(off[3] + rows * kmax * 8);                 // nkept
  off[5] = align256(off[4] + rows * 4);                        // counts
  off[6] = align256(off[5] + nb * 4);                          // offsets
  off[7] = align256(off[6] + nb * 4);                          // pairs
  off[8] = align256(off[7] + rows * kmax * 8);                 // tree levels
  off[9] = align256(off[8] + (prefill_tree_supported(p) ? prefill_tree_workspace_need(p, n_q) : 0));
  if (total) *total = off[9];
  LeafPaths lp = {};
  if (ws) {
    char* base = reinterpret_cast<char*>(ws);
    lp.part = reinterpret_cast<float*>(base + off[0]);
    lp.lpart = reinterpret_cast<float*>(base + off[1]);
    lp.lml = reinterpret_cast<float2*>(base + off[2]);
    lp.kept = reinterpret_cast<int2*>(base + off[3]);
    lp.nkept = reinterpret_cast<int*>(base + off[4]);
    lp.counts = reinterpret_cast<int*>(base + off[5]);
    lp.offsets = reinterpret_cast<int*>(base + off[6]);
    lp.pairs = reinterpret_cast<int2*>(base + off[7]);
    lp.tree_ws = prefill_tree_supported(p) ? base + off[8] : nullptr;
  }
  return lp;
}

// Exclusive prefix sum of n counts, one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(const int* __restrict__ counts,
                                                    int* __restrict__ offsets, int64_t n) {
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x;
  const int64_t per = (n + 1023) / 1024;
  const int64_t b0 = int64_t(tid) * per;
  const int64_t b1 = b0 + per < n ? b0 + per : n;
  int s = 0;
  for (int64_t i = b0; i < b1; ++i) s += counts[i];
  // inclusive scan of the per-thread sums
  int x = s;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  int run = x - s + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int64_t i = b0; i < b1; ++i) {
    offsets[i] = run;
    run += counts[i];
  }
}

// Query rotation index of slot s: n0 - 1 - s B, n0 = kept * B + window tokens.
__device__ __forceinline__ int64_t window_tokens(const Params& p, int64_t t) {
  const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
  return t + 1 - (s0 / p.B) * p.B;
}

__global__ void scatter_kernel(Params p, LeafPaths lp, int64_t q_start, int n_q, int kmax) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rows = int64_t(p.batch) * n_q * p.hq;
  if (i >= rows * kmax) return;
  const int64_t row = i / kmax;
  const int s = int(i % kmax);
  const int nk = lp.nkept[row];
  if (s >= nk) return;
  const int2 rec = lp.kept[i];
  const int64_t qi = (row / p.hq) % n_q;
  const int64_t t = q_start + qi;
  const int64_t n0 = int64_t(nk) * p.B + window_tokens(p, t);
  const int rot = int(n0 - 1 - int64_t(s) * p.B);
  lp.pairs[lp.offsets[rec.x] + rec.y] = make_int2(int(row), (s << 24) | rot);
}

// Shared-memory operand tiles of leaf_tc_kernel (TF32, K-major, no swizzle).
// NS = 2 keeps each operand twice, as the high and the low TF32 parts of its
// fp32 value (the split-operand "3xTF32" scheme: x = hi + lo, and
// A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi recovers fp32 accuracy from
// TF32 products); NS = 1 keeps the TF32 rounding alone.
template <int D, int BL, int NS>
struct LeafSmem {
  static constexpr int kA1n = kTile * D * 4, kB1n = BL * D * 4;     // bytes of one part
  static constexpr int kA2n = kTile * BL * 4, kB2n = D * BL * 4;
  static constexpr int kA1 = 0;                       // queries   [128][D]  (x NS)
  static constexpr int kB1 = kA1 + NS * kA1n;         // keys      [BL][D]
  static constexpr int kA2 = kB1 + NS * kB1n;         // probs     [128][BL]
  static constexpr int kB2 = kA2 + NS * kA2n;         // values^T  [D][BL]
  static constexpr int kDst = kB2 + NS * kB2n;        // per tile row: partial offset
  static constexpr int kBar = kDst + kTile * 8;       // 2 mbarriers + TMEM address
  static constexpr int kTotal = kBar + 32;
  static constexpr bool kFits = kTotal <= 227 * 1024;
};

// Element (r, k) of a K-major no-swizzle fp32 operand with R rows: byte offset.
__device__ __forceinline__ int kmaj(int R, int r, int k) { return (k >> 2) * 16 * R + r * 16 + (k & 3) * 4; }

template <typename T>
__device__ __forceinline__ void load8(const T* src, float* v);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* src, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load1(const float* p) { return *p; }

// Store 4 values TF32-rounded at `dst`; with a split (lo_off != 0) also the
// TF32 rounding of what the first rounding left, lo_off bytes further.
__device__ __forceinline__ void store4(unsigned char* dst, int lo_off, float a, float b, float c,
                                       float d) {
  const float ha = tc05::to_tf32(a), hb = tc05::to_tf32(b), hc = tc05::to_tf32(c),
              hd = tc05::to_tf32(d);
  *reinterpret_cast<float4*>(dst) = make_float4(ha, hb, hc, hd);
  if (lo_off)
    *reinterpret_cast<float4*>(dst + lo_off) =
        make_float4(tc05::to_tf32(a - ha), tc05::to_tf32(b - hb), tc05::to_tf32(c - hc),
                    tc05::to_tf32(d - hd));
}

// Rotate 8 rotate-half pairs (x1[c], x2[c]) at frequencies j0 .. j0+7 by table
// row `row_idx` and store them as two 8-element runs of operand row r.
__device__ __forceinline__ void rotate_store(const Params& p, const float2* rope, int row_idx,
                                             int j0, const float* x1, const float* x2,
                                             unsigned char* base, int lo_off, int R, int r) {
  const int half = p.d / 2;
  float y1[8], y2[8];
  if (p.rope) {
    const float4* cs = reinterpret_cast<const float4*>(rope + int64_t(row_idx) * half + j0);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 v = cs[c];   // (cos, sin) of j0 + 2c and j0 + 2c + 1
      y1[2 * c] = x1[2 * c] * v.x - x2[2 * c] * v.y;
      y2[2 * c] = x2[2 * c] * v.x + x1[2 * c] * v.y;
      y1[2 * c + 1] = x1[2 * c + 1] * v.z - x2[2 * c + 1] * v.w;
      y2[2 * c + 1] = x2[2 * c + 1] * v.z + x1[2 * c + 1] * v.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      y1[c] = x1[c];
      y2[c] = x2[c];
    }
  }
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    store4(base + kmaj(R, r, j0 + 4 * c), lo_off, y1[4 * c], y1[4 * c + 1], y1[4 * c + 2],
           y1[4 * c + 3]);
    store4(base + kmaj(R, r, half + j0 + 4 * c), lo_off, y2[4 * c], y2[4 * c + 1],
           y2[4 * c + 2], y2[4 * c + 3]);
  }
}

// One CTA per leaf bucket (sequence, KV head, leaf): the leaf's keys (rotated
// by their offset in the leaf) and values are staged once, then its pairs run
// in tiles of 128: S = Q_rot K_rot^T on tcgen05 into TMEM, a per-row softmax
// in registers (thread i owns pair i), O = P V on tcgen05, and the pair's
// partial (normalised output, max, sum) is written out.
template <typename T, int D, int BL, int NS>
__global__ void __launch_bounds__(kLThreads, 2)
leaf_tc_kernel(Params p, const T* __restrict__ Q, const T* __restrict__ K,
               const T* __restrict__ V, void* tree, LeafPaths lp, int kmax, int nleaf) {
  using L = LeafSmem<D, BL, NS>;
  constexpr int HALF = D / 2;
  constexpr int TCOLS = 256;          // S in columns [0, BL), O in [128, 128 + D)
  const int64_t b = blockIdx.x;
  const int cnt = lp.counts[b];
  if (cnt == 0) return;
  const int off = lp.offsets[b];
  const int64_t seq = b / (int64_t(p.hkv) * nleaf);
  const int g = int((b / nleaf) % p.hkv);
  const int leaf = int(b % nleaf);

  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kBar + 16);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (warp == 0) {
    tc05::tmem_alloc(tslot, TCOLS);
    tc05::tmem_relinquish();
  }
  if (tid == 0) {
    tc05::mbar_init(&bar[0], 1);
    tc05::mbar_init(&bar[1], 1);
    tc05::mbar_fence_init();
  }
  const float2* rope = rope_table(p, tree);

  // the leaf's keys rotated by their offset j, and its values transposed
  const int64_t row0 = ((seq * p.hkv + g) * p.cap + int64_t(leaf) * BL);
  for (int task = tid; task < BL * (HALF / 8); task += kLThreads) {
    const int j = task % BL, c = task / BL;
    float x1[8], x2[8];
    load8<T>(K + (row0 + j) * D + 8 * c, x1);
    load8<T>(K + (row0 + j) * D + HALF + 8 * c, x2);
    rotate_store(p, rope, j, 8 * c, x1, x2, sm + L::kB1, NS > 1 ? L::kB1n : 0, BL, j);
  }
  for (int task = tid; task < D * (BL / 4); task += kLThreads) {
    const int n = task % D, kq = task / D;
    float4 v;
    v.x = load1(V + (row0 + 4 * kq + 0) * D + n);
    v.y = load1(V + (row0 + 4 * kq + 1) * D + n);
    v.z = load1(V + (row0 + 4 * kq + 2) * D + n);
    v.w = load1(V + (row0 + 4 * kq + 3) * D + n);
    store4(sm + L::kB2 + kmaj(D, n, 4 * kq), NS > 1 ? L::kB2n : 0, v.x, v.y, v.z, v.w);
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t aA1 = tc05::smem_u32(sm + L::kA1), aB1 = tc05::smem_u32(sm + L::kB1);
  const uint32_t aA2 = tc05::smem_u32(sm + L::kA2), aB2 = tc05::smem_u32(sm + L::kB2);
  constexpr uint32_t id1 = tc05::idesc(tc05::kFmtTF32, kTile, BL);
  constexpr uint32_t id2 = tc05::idesc(tc05::kFmtTF32, kTile, D);
  const float inv_sqrt_d = p.inv_sqrt_d;
  bool ok = true;
  unsigned phase = 0;

  for (int t0 = 0; t0 < cnt && ok; t0 += kTile) {
    const int nt = cnt - t0 < kTile ? cnt - t0 : kTile;
    // gather and rotate the tile's queries (rows past nt are zero); every load
    // of this thread's tasks is issued before any store
    constexpr int NT = kTile * (HALF / 8) / kLThreads;
    int2 prs[NT];
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int r = (tid + it * kLThreads) % kTile;
      prs[it] = r < nt ? lp.pairs[off + t0 + r] : make_int2(0, 0);
    }
    float xa[NT][8], xb[NT][8];
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int task = tid + it * kLThreads;
      const int r = task % kTile, c = task / kTile;
      if (r < nt) {
        const T* q = Q + int64_t(prs[it].x) * D;
        load8<T>(q + 8 * c, xa[it]);
        load8<T>(q + HALF + 8 * c, xb[it]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xa[it][e] = xb[it][e] = 0.f;
      }
    }
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int task = tid + it * kLThreads;
      const int r = task % kTile, c = task / kTile;
      const int rot = r < nt ? (prs[it].y & 0xffffff) : 0;
      rotate_store(p, rope, rot, 8 * c, xa[it], xb[it], sm + L::kA1, NS > 1 ? L::kA1n : 0,
                   kTile, r);
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const uint32_t a = aA1 + kk * 32 * kTile, b = aB1 + kk * 32 * BL;
        tc05::mma_tf32(tS, tc05::desc_kmajor(a, 16 * kTile, 128),
                       tc05::desc_kmajor(b, 16 * BL, 128), id1, kk > 0);
        if (NS > 1) {   // + hi * lo + lo * hi
          tc05::mma_tf32(tS, tc05::desc_kmajor(a, 16 * kTile, 128),
                         tc05::desc_kmajor(b + L::kB1n, 16 * BL, 128), id1, 1);
          tc05::mma_tf32(tS, tc05::desc_kmajor(a + L::kA1n, 16 * kTile, 128),
                         tc05::desc_kmajor(b, 16 * BL, 128), id1, 1);
        }
      }
      tc05::mma_commit(&bar[0]);
    }
    ok = __syncthreads_and(tid != 0 || tc05::mbar_wait_bounded(&bar[0], phase, kLeafWaitNs));
    tc05::fence_after_sync();
    // M = 64 accumulators: row 16 w + i sits in TMEM lane 32 w + i (i < 16);
    // lane i < 16 of warp w owns that row, the other lanes take part in the
    // warp-collective loads only
    const int lane = tid & 31;
    const int myrow = 16 * warp + lane;
    const bool rowthr = lane < 16;
    float m = -INFINITY, l = 0.f;
    if (ok) {
      float s[BL];
#pragma unroll
      for (int c = 0; c < BL / 16; ++c)
        tc05::tmem_ld16(tS + (uint32_t(warp * 32) << 16) + 16 * c, s + 16 * c);
      tc05::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < BL; ++c) {
        s[c] *= inv_sqrt_d;
        m = fmaxf(m, s[c]);
      }
#pragma unroll
      for (int c = 0; c < BL; ++c) {
        s[c] = __expf(s[c] - m);
        l += s[c];
      }
      if (rowthr) {
#pragma unroll
        for (int c = 0; c < BL; c += 4)
          store4(sm + L::kA2 + kmaj(kTile, myrow, c), NS > 1 ? L::kA2n : 0, s[c], s[c + 1],
                 s[c + 2], s[c + 3]);
      }
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (tid == 0 && ok) {
#pragma unroll
      for (int kk = 0; kk < BL / 8; ++kk) {
        const uint32_t a = aA2 + kk * 32 * kTile, b = aB2 + kk * 32 * D;
        tc05::mma_tf32(tO, tc05::desc_kmajor(a, 16 * kTile, 128),
                       tc05::desc_kmajor(b, 16 * D, 128), id2, kk > 0);
        if (NS > 1) {
          tc05::mma_tf32(tO, tc05::desc_kmajor(a, 16 * kTile, 128),
                         tc05::desc_kmajor(b + L::kB2n, 16 * D, 128), id2, 1);
          tc05::mma_tf32(tO, tc05::desc_kmajor(a + L::kA2n, 16 * kTile, 128),
                         tc05::desc_kmajor(b, 16 * D, 128), id2, 1);
        }
      }
      tc05::mma_commit(&bar[1]);
    }
    ok = __syncthreads_and(tid != 0 || !ok || tc05::mbar_wait_bounded(&bar[1], phase, kLeafWaitNs)) && ok;
    tc05::fence_after_sync();
    // O rows: the row's owner reads it from TMEM (warp-collective loads:
    // every lane loads) into a staging copy in the query tile's bytes (free
    // since the first product completed), 16-byte chunks rotated by the row so
    // that the writes spread over the banks; then every warp stores whole
    // rows, coalesced
    constexpr int CPR = D / 4;                     // 16-byte chunks per row
    unsigned char* stg = sm + L::kA1;
    static_assert(kTile * D * 4 <= L::kA1n, "staging fits the query tile");
    if (ok) {
      const float il = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc05::tmem_ld16(tO + (uint32_t(warp * 32) << 16) + 32 * c, o);
        tc05::tmem_ld16(tO + (uint32_t(warp * 32) << 16) + 32 * c + 16, o + 16);
        tc05::tmem_wait_ld();
        if (rowthr) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = 8 * c + e;
            *reinterpret_cast<float4*>(stg + myrow * (D * 4) + ((ch + myrow) % CPR) * 16) =
                make_float4(o[4 * e] * il, o[4 * e + 1] * il, o[4 * e + 2] * il,
                            o[4 * e + 3] * il);
          }
        }
      }
      if (rowthr && myrow < nt) {
        const int2 pr = lp.pairs[off + t0 + myrow];
        const int64_t slot = int64_t(pr.x) * kmax + (pr.y >> 24);
        lp.lml[slot] = make_float2(m, l);
        reinterpret_cast<int64_t*>(sm + L::kDst)[myrow] = slot * D;
      }
    }
    __syncthreads();
    if (ok) {
      // destination rows from shared memory: no global load between the stores
      constexpr int RPW = 32 / CPR;                  // rows per warp instruction
      const int sub = (threadIdx.x & 31) / CPR, ch = (threadIdx.x & 31) % CPR;
      const int64_t* dsts = reinterpret_cast<const int64_t*>(sm + L::kDst);
      for (int r = warp * RPW + sub; r < nt; r += (kLThreads / 32) * RPW) {
        float* dst = lp.lpart + dsts[r];
        *reinterpret_cast<float4*>(dst + 4 * ch) =
            *reinterpret_cast<const float4*>(stg + r * (D * 4) + ((ch + r) % CPR) * 16);
      }
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    phase ^= 1u;
  }
  if (!ok && tid == 0) {
    atomicOr(tree_error_word(tree), RECSA_DEVERR_WAIT_TIMEOUT);
    // let the MMAs still in flight finish before the columns are released
    tc05::mbar_wait_bounded(&bar[0], phase, kLeafWaitNs);
    tc05::mbar_wait_bounded(&bar[1], phase, kLeafWaitNs);
  }
  __syncthreads();
  if (warp == 0) tc05::tmem_dealloc(tmem, TCOLS);
}

// Per query head: the traversal's partial (window and unselected summaries)
// merged with its kept leaves' partials; one warp per query head.
template <typename T, int D>
__global__ void merge_kernel(Params p, LeafPaths lp, int64_t rows, int kmax, T* __restrict__ O) {
  constexpr int PER = D / 32;
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* pr = lp.part + row * (D + 2);
  float acc[PER];
  float2 ml = *reinterpret_cast<const float2*>(pr + D);
  float M = ml.x, Lsum = ml.y;
#pragma unroll
  for (int c = 0; c < PER; ++c) acc[c] = pr[lane * PER + c] * ml.y;
  const int nk = lp.nkept[row];
  for (int s = 0; s < nk; ++s) {
    const float* q = lp.lpart + (row * kmax + s) * D;
    const float2 ms = lp.lml[row * kmax + s];
    const float mn = fmaxf(M, ms.x);
    const float ra = M == -INFINITY ? 0.f : __expf(M - mn);
    const float rb = __expf(ms.x - mn) * ms.y;
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[c] = acc[c] * ra + q[lane * PER + c] * rb;
    Lsum = Lsum * ra + rb;
    M = mn;
  }
  const float il = 1.f / Lsum;
#pragma unroll
  for (int c = 0; c < PER; ++c) store_elem(O, row * D + lane * PER + c, acc[c] * il,
                                           sizeof(T) == 2 ? RECSA_DTYPE_BF16 : RECSA_DTYPE_F32);
}

template <typename T, int D, int BL>
cudaError_t leaf_typed(const Params& p, const void* Q, const void* K, const void* V, void* tree,
                       const LeafPaths& lp, int kmax, cudaStream_t s) {
  // fp32 inputs: split operands (fp32 accuracy); bf16 inputs are exact in TF32
  // and their rotations and probabilities need no more than its rounding
  constexpr int NS = sizeof(T) == 4 ? 2 : 1;
  using L = LeafSmem<D, BL, NS>;
  if constexpr (!L::kFits) {
    return cudaErrorNotSupported;
  } else {
    auto kern = leaf_tc_kernel<T, D, BL, NS>;
    cudaError_t e = ensure_smem(kern, L::kTotal);
    if (e != cudaSuccess) return e;
    const int nleaf = int(p.lay.nodes[0]);
    kern<<<unsigned(buckets_of(p)), kLThreads, L::kTotal, s>>>(
        p, reinterpret_cast<const T*>(Q), reinterpret_cast<const T*>(K),
        reinterpret_cast<const T*>(V), tree, lp, kmax, nleaf);
    return cudaGetLastError();
  }
}

template <typename T, int D>
cudaError_t leaf_dispatch(const Params& p, const void* Q, const void* K, const void* V,
                          void* tree, const LeafPaths& lp, int kmax, cudaStream_t s) {
  switch (p.B) {
    case 16: return leaf_typed<T, D, 16>(p, Q, K, V, tree, lp, kmax, s);
    case 32: return leaf_typed<T, D, 32>(p, Q, K, V, tree, lp, kmax, s);
    case 64: return leaf_typed<T, D, 64>(p, Q, K, V, tree, lp, kmax, s);
  }
  return cudaErrorNotSupported;
}

bool leaf_fits(const Params& p) {
  const bool split = p.dtype != RECSA_DTYPE_BF16;
  auto fits = [&](auto d, auto bl) {
    constexpr int Dv = decltype(d)::value, BLv = decltype(bl)::value;
    return split ? LeafSmem<Dv, BLv, 2>::kFits : LeafSmem<Dv, BLv, 1>::kFits;
  };
  using I64 = std::integral_constant<int, 64>;
  using I128 = std::integral_constant<int, 128>;
  using B16 = std::integral_constant<int, 16>;
  using B32 = std::integral_constant<int, 32>;
  using B64 = std::integral_constant<int, 64>;
  if (p.d == 64) return p.B == 16 ? fits(I64{}, B16{}) : p.B == 32 ? fits(I64{}, B32{}) : fits(I64{}, B64{});
  return p.B == 16 ? fits(I128{}, B16{}) : p.B == 32 ? fits(I128{}, B32{}) : fits(I128{}, B64{});
}

}  // namespace

bool prefill_tc_supported(const Params& p) {
  if (p.mode != RECSA_MODE_RECSA) return false;
  if (p.d != 64 && p.d != 128) return false;
  if (p.B != 16 && p.B != 32 && p.B != 64) return false;
  if (!leaf_fits(p)) return false;
  if (p.lay.levels < 1) return false;
  if (kmax_of(p) > 64) return false;
  if (buckets_of(p) > 0x7fffffff) return false;
  // query rotations are packed in 24 bits
  if (int64_t(p.B) * kmax_of(p) + p.W + p.B >= (int64_t(1) << 24)) return false;
  return true;
}

size_t prefill_tc_workspace_need(const Params& p, int32_t n_q) {
  size_t total = 0;
  carve(p, n_q, nullptr, &total);
  return total;
}

cudaError_t launch_prefill_tc(const Params& p, const void* Q, const void* K, const void* V,
                              const void* tree, int64_t q_start, int32_t n_q, void* O,
                              int32_t* trace, void* ws, cudaStream_t s) {
  if (!prefill_tc_supported(p)) return cudaErrorNotSupported;
  const LeafPaths lp = carve(p, n_q, ws, nullptr);
  const int kmax = kmax_of(p);
  const int64_t nb = buckets_of(p);
  const int64_t rows = int64_t(p.batch) * n_q * p.hq;
  cudaError_t e = cudaMemsetAsync(lp.counts, 0, size_t(nb) * 4, s);
  if (e != cudaSuccess) return e;
  // 1. window partials (bf16 on the window kernel; otherwise the traversal attends it)
  const float* wpart = nullptr;
  e = launch_prefill_window(p, Q, K, V, tree, q_start, n_q, lp.part, s);
  if (e == cudaSuccess) {
    wpart = lp.part;
  } else if (e == cudaErrorNotSupported) {
    cudaGetLastError();
  } else {
    return e;
  }
  // 2. traversal: summaries + window into lp.part, kept leaves, per-leaf counts;
  // by parent-node tiles on the tensor cores (needs the window partials), else
  // by the warp-per-query-head kernel
  LeafOut lo;
  lo.part = lp.part;
  lo.kept = lp.kept;
  lo.nkept = lp.nkept;
  lo.counts = lp.counts;
  lo.nleaf = int(p.lay.nodes[0]);
  lo.kmax = kmax;
  e = cudaErrorNotSupported;
  if (wpart && lp.tree_ws && switches().prefill_path != 2)
    e = launch_prefill_tree(p, Q, tree, q_start, n_q, trace, lo, lp.tree_ws, s);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    e = launch_prefill_warp_leafout(p, Q, K, V, tree, q_start, n_q, trace, wpart, lo, s);
  }
  if (e != cudaSuccess) return e;
  // 3. offsets, 4. pairs grouped by leaf
  scan_kernel<<<1, 1024, 0, s>>>(lp.counts, lp.offsets, nb);
  const int64_t tasks = rows * kmax;
  scatter_kernel<<<unsigned((tasks + 255) / 256), 256, 0, s>>>(p, lp, q_start, n_q, kmax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 5. kept-leaf partials on the tensor cores
  void* tr = const_cast<void*>(tree);
  if (p.dtype == RECSA_DTYPE_BF16)
    e = p.d == 128 ? leaf_dispatch<__nv_bfloat16, 128>(p, Q, K, V, tr, lp, kmax, s)
                   : leaf_dispatch<__nv_bfloat16, 64>(p, Q, K, V, tr, lp, kmax, s);
  else
    e = p.d == 128 ? leaf_dispatch<float, 128>(p, Q, K, V, tr, lp, kmax, s)
                   : leaf_dispatch<float, 64>(p, Q, K, V, tr, lp, kmax, s);
  if (e != cudaSuccess) return e;
  // 6. merge into O
  const unsigned mblocks = unsigned((rows + 7) / 8);
  if (p.dtype == RECSA_DTYPE_BF16) {
    if (p.d == 128)
      merge_kernel<__nv_bfloat16, 128><<<mblocks, 256, 0, s>>>(p, lp, rows, kmax,
                                                              reinterpret_cast<__nv_bfloat16*>(O));
    else
      merge_kernel<__nv_bfloat16, 64><<<mblocks, 256, 0, s>>>(p, lp, rows, kmax,
                                                             reinterpret_cast<__nv_bfloat16*>(O));
  } else {
    if (p.d == 128)
      merge_kernel<float, 128><<<mblocks, 256, 0, s>>>(p, lp, rows, kmax,
                                                      reinterpret_cast<float*>(O));
    else
      merge_kernel<float, 64><<<mblocks, 256, 0, s>>>(p, lp, rows, kmax,
                                                     reinterpret_cast<float*>(O));
  }
  return cudaGetLastError();
}

}  // namespace recsa
