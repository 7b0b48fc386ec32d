// Prefill, exact local window on the fifth-generation tensor cores (tcgen05).
//
// For a query at t the window is [a B, t] (a = floor(max(0, t + 1 - W) / B)),
// and the RoPE angle between the query and a window token is the true
// distance t - pos ("Recursive Sparse Attention: Million-Token Length
// Extrapolation at Logarithmic Cost", abstract: candidate-local positions; the
// window keeps its order after the kept leaves' tokens).  Consecutive queries
// share most of their windows, so the window is a banded causal attention over
// query blocks: a CTA takes 128 rows (128 / G consecutive queries x the G heads
// of one KV group) and walks the union of their windows in blocks of 64 keys.
// Per block: the keys, rotated to a CTA-local origin, and the values are
// staged as TF32 operands; S = Q K^T is one [128 x d] x [d x 64] tcgen05
// product into TMEM; each row's band mask and online softmax run in registers
// (thread i of warps 0-3 owns row i); P V is a second product, read back and
// added to the row's fp32 output.  The result is the window's partial softmax
// (normalised output, max, sum) per query head, the same rows the tree pass
// folds the summaries and kept leaves into.  The queries and keys are bf16
// (exact in TF32); only their fp32 rotations and the probabilities are
// rounded, to TF32.
#include "recsa_internal.cuh"
#include "tc05.cuh"

namespace recsa {
namespace {

constexpr int kWRows = 128;       // query rows per CTA (MMA M)
constexpr int kWKeys = 64;        // keys per block (MMA N of the scores)
constexpr int kWThreads2 = 256;
constexpr unsigned long long kWinWaitNs = 200000000ull;

template <int D>
struct WinSmem {
  static constexpr int kA1 = 0;                              // queries  [128][D]
  static constexpr int kB1 = kA1 + kWRows * D * 4;           // keys     [64][D]
  static constexpr int kA2 = kB1 + kWKeys * D * 4;           // probs    [128][64]
  static constexpr int kB2 = kA2 + kWRows * kWKeys * 4;      // values^T [D][64]
  static constexpr int kBar = kB2 + D * kWKeys * 4;
  static constexpr int kTotal = kBar + 32;
  static_assert(kTotal <= 227 * 1024, "window tile does not fit");
};

__device__ __forceinline__ int kmw(int R, int r, int k) { return (k >> 2) * 16 * R + r * 16 + (k & 3) * 4; }

// rotate 8 rotate-half pairs (bf16 at src, src + D/2) by table row idx, store
// them TF32-rounded as row r of a K-major operand of R rows
template <int D>
__device__ __forceinline__ void rot8_store(const __nv_bfloat16* src, const float2* rope, int rope_on,
                                           int idx, int j0, unsigned char* base, int R, int r,
                                           bool zero) {
  constexpr int HALF = D / 2;
  float x1[8], x2[8];
  if (!zero) {
    const uint4 u1 = *reinterpret_cast<const uint4*>(src + j0);
    const uint4 u2 = *reinterpret_cast<const uint4*>(src + HALF + j0);
    const uint32_t w1[4] = {u1.x, u1.y, u1.z, u1.w}, w2[4] = {u2.x, u2.y, u2.z, u2.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x1[2 * e] = __uint_as_float(w1[e] << 16);
      x1[2 * e + 1] = __uint_as_float(w1[e] & 0xffff0000u);
      x2[2 * e] = __uint_as_float(w2[e] << 16);
      x2[2 * e + 1] = __uint_as_float(w2[e] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x1[e] = x2[e] = 0.f;
  }
  float y1[8], y2[8];
  if (rope_on && !zero) {
    const float4* cs = reinterpret_cast<const float4*>(rope + int64_t(idx) * HALF + j0);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 v = cs[c];
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
    *reinterpret_cast<float4*>(base + kmw(R, r, j0 + 4 * c)) =
        make_float4(tc05::to_tf32(y1[4 * c]), tc05::to_tf32(y1[4 * c + 1]),
                    tc05::to_tf32(y1[4 * c + 2]), tc05::to_tf32(y1[4 * c + 3]));
    *reinterpret_cast<float4*>(base + kmw(R, r, HALF + j0 + 4 * c)) =
        make_float4(tc05::to_tf32(y2[4 * c]), tc05::to_tf32(y2[4 * c + 1]),
                    tc05::to_tf32(y2[4 * c + 2]), tc05::to_tf32(y2[4 * c + 3]));
  }
}

template <int D>
__global__ void __launch_bounds__(kWThreads2, 1)
window_tc_kernel(Params p, const __nv_bfloat16* __restrict__ Q,
                 const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                 void* tree, int64_t q_start, int n_q, float* __restrict__ part) {
  using S = WinSmem<D>;
  constexpr int HALF = D / 2;
  const int G = p.group, QB = kWRows / G;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t seq = blockIdx.y / p.hkv;
  const int g = int(blockIdx.y % p.hkv);
  const int q0 = blockIdx.x * QB;
  const int nqh = min(QB, n_q - q0);
  const int64_t t0 = q_start + q0;
  auto win_lo = [&](int64_t t) -> int64_t {
    const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
    return s0 / p.B * p.B;
  };
  const int64_t base = win_lo(t0);                  // CTA-local RoPE origin
  const int64_t kend = t0 + nqh;                    // one past the last key
  const int nblk = int((kend - base + kWKeys - 1) / kWKeys);

  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + S::kBar + 16);
  constexpr uint32_t kCols = 256;                   // S in [0, 64), P V in [128, 128 + D)
  if (warp == 0) {
    tc05::tmem_alloc(tslot, kCols);
    tc05::tmem_relinquish();
  }
  if (tid == 0) {
    tc05::mbar_init(&bar[0], 1);
    tc05::mbar_init(&bar[1], 1);
    tc05::mbar_fence_init();
  }
  const float2* rope = rope_table(p, tree);
  // query rows (query qq = row / G, head g G + row % G) rotated by t - base
  for (int task = tid; task < kWRows * (HALF / 8); task += kWThreads2) {
    const int r = task % kWRows, c = task / kWRows;
    const int qq = r / G, hh = r % G;
    const bool zero = qq >= nqh;
    const __nv_bfloat16* src =
        Q + ((seq * n_q + q0 + (zero ? 0 : qq)) * p.hq + int64_t(g) * G + hh) * D;
    rot8_store<D>(src, rope, p.rope, int(t0 + qq - base), 8 * c, sm + S::kA1, kWRows, r, zero);
  }
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  const uint32_t aA1 = tc05::smem_u32(sm + S::kA1), aB1 = tc05::smem_u32(sm + S::kB1);
  const uint32_t aA2 = tc05::smem_u32(sm + S::kA2), aB2 = tc05::smem_u32(sm + S::kB2);
  constexpr uint32_t id1 = tc05::idesc(tc05::kFmtTF32, kWRows, kWKeys);
  constexpr uint32_t id2 = tc05::idesc(tc05::kFmtTF32, kWRows, D);
  const float inv_sqrt_d = p.inv_sqrt_d;
  // this thread's row (warps 0-3)
  const int myqq = (tid < kWRows) ? tid / G : QB;
  const int lo = myqq < nqh ? int(win_lo(t0 + myqq) - base) : 1 << 30;
  const int hi = myqq < nqh ? int(t0 + myqq - base) : -1;
  float o[D];
#pragma unroll
  for (int e = 0; e < D; ++e) o[e] = 0.f;
  float m = -INFINITY, l = 0.f;
  bool ok = true;
  unsigned phase = 0;
  uint32_t tmem = 0;
  for (int kb = 0; kb < nblk && ok; ++kb) {
    const int64_t k0 = base + int64_t(kb) * kWKeys;
    if (kb > 0) {
      // the previous block's products are done: its operands may be replaced
      tc05::fence_before_sync();
      __syncthreads();
      tc05::fence_after_sync();
    }
    for (int task = tid; task < kWKeys * (HALF / 8); task += kWThreads2) {
      const int j = task % kWKeys, c = task / kWKeys;
      const bool zero = k0 + j >= kend;
      rot8_store<D>(K + (kvbase + (zero ? 0 : k0 + j)) * D, rope, p.rope, int(k0 + j - base),
                    8 * c, sm + S::kB1, kWKeys, j, zero);
    }
    for (int task = tid; task < D * (kWKeys / 4); task += kWThreads2) {
      const int n = task % D, kq = task / D;
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t pos = k0 + 4 * kq + e;
        v[e] = pos < kend ? __bfloat162float(V[(kvbase + pos) * D + n]) : 0.f;
      }
      *reinterpret_cast<float4*>(sm + S::kB2 + kmw(D, n, 4 * kq)) =
          make_float4(tc05::to_tf32(v[0]), tc05::to_tf32(v[1]), tc05::to_tf32(v[2]),
                      tc05::to_tf32(v[3]));
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    tmem = *tslot;
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk)
        tc05::mma_tf32(tmem, tc05::desc_kmajor(aA1 + kk * 32 * kWRows, 16 * kWRows, 128),
                       tc05::desc_kmajor(aB1 + kk * 32 * kWKeys, 16 * kWKeys, 128), id1, kk > 0);
      tc05::mma_commit(&bar[0]);
    }
    ok = __syncthreads_and(tid != 0 || tc05::mbar_wait_bounded(&bar[0], phase, kWinWaitNs));
    tc05::fence_after_sync();
    float scale = 1.f;
    if (warp < 4 && ok) {
      // every lane loads (warp-collective); rows past the block mask to zero
      float s[kWKeys];
#pragma unroll
      for (int c = 0; c < kWKeys / 16; ++c)
        tc05::tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + 16 * c, s + 16 * c);
      tc05::tmem_wait_ld();
      const int kbase = int(k0 - base);
      float bm = -INFINITY;
#pragma unroll
      for (int c = 0; c < kWKeys; ++c) {
        const int kk = kbase + c;
        const bool in = kk >= lo && kk <= hi;
        s[c] = in ? s[c] * inv_sqrt_d : -INFINITY;
        bm = fmaxf(bm, s[c]);
      }
      const float mn = fmaxf(m, bm);
      scale = (m == -INFINITY) ? 0.f : __expf(m - mn);
      float bl = 0.f;
#pragma unroll
      for (int c = 0; c < kWKeys; ++c) {
        s[c] = (s[c] == -INFINITY) ? 0.f : __expf(s[c] - mn);
        bl += s[c];
      }
      if (mn != -INFINITY) {
        l = l * scale + bl;
        m = mn;
      } else {
        scale = 1.f;
      }
#pragma unroll
      for (int c = 0; c < kWKeys; c += 4)
        *reinterpret_cast<float4*>(sm + S::kA2 + kmw(kWRows, tid, c)) =
            make_float4(tc05::to_tf32(s[c]), tc05::to_tf32(s[c + 1]), tc05::to_tf32(s[c + 2]),
                        tc05::to_tf32(s[c + 3]));
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (tid == 0 && ok) {
#pragma unroll
      for (int kk = 0; kk < kWKeys / 8; ++kk)
        tc05::mma_tf32(tmem + 128, tc05::desc_kmajor(aA2 + kk * 32 * kWRows, 16 * kWRows, 128),
                       tc05::desc_kmajor(aB2 + kk * 32 * D, 16 * D, 128), id2, kk > 0);
      tc05::mma_commit(&bar[1]);
    }
    ok = __syncthreads_and(tid != 0 || !ok || tc05::mbar_wait_bounded(&bar[1], phase, kWinWaitNs)) && ok;
    tc05::fence_after_sync();
    if (warp < 4 && ok) {
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        float x[16];
        tc05::tmem_ld16(tmem + 128 + (uint32_t(warp * 32) << 16) + 16 * c, x);
        tc05::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o[16 * c + e] = o[16 * c + e] * scale + x[e];
      }
    }
    phase ^= 1u;
  }
  if (!ok && tid == 0) {
    atomicOr(tree_error_word(tree), RECSA_DEVERR_WAIT_TIMEOUT);
    tc05::mbar_wait_bounded(&bar[0], phase, kWinWaitNs);
    tc05::mbar_wait_bounded(&bar[1], phase, kWinWaitNs);
  }
  // partial row per (query, head): normalised output, max, sum
  if (tid < kWRows && myqq < nqh && ok) {
    const int hh = tid % G;
    float* row = part + ((seq * n_q + q0 + myqq) * p.hq + int64_t(g) * G + hh) * (D + 2);
    const float il = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < D; e += 2)
      *reinterpret_cast<float2*>(row + e) = make_float2(o[e] * il, o[e + 1] * il);
    *reinterpret_cast<float2*>(row + D) = make_float2(m, l);
  }
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc05::tmem_dealloc(*tslot, kCols);
}

}  // namespace

// The tensor-core window kernel; cudaErrorNotSupported outside its limits
// (bf16; G divides 128; the RoPE table reaches W + B + 128 / G indices).
cudaError_t launch_prefill_window_tc(const Params& p, const void* Q, const void* K,
                                     const void* V, const void* tree, int64_t q_start,
                                     int32_t n_q, void* part, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA && p.mode != RECSA_MODE_ZHA) return cudaErrorNotSupported;
  if (p.dtype != RECSA_DTYPE_BF16 || (p.d != 64 && p.d != 128)) return cudaErrorNotSupported;
  if (p.group < 1 || kWRows % p.group) return cudaErrorNotSupported;
  const int QB = kWRows / p.group;
  if (p.rope && int64_t(p.W) + p.B + QB > p.lay.rope_rows) return cudaErrorNotSupported;
  if (int64_t(p.batch) * p.hkv > 65535) return cudaErrorNotSupported;
  dim3 grid(unsigned((n_q + QB - 1) / QB), unsigned(p.batch * p.hkv));
  cudaError_t e;
  if (p.d == 128) {
    auto kern = window_tc_kernel<128>;
    e = ensure_smem(kern, WinSmem<128>::kTotal);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWThreads2, WinSmem<128>::kTotal, s>>>(
        p, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
        const_cast<void*>(tree), q_start, n_q, (float*)part);
  } else {
    auto kern = window_tc_kernel<64>;
    e = ensure_smem(kern, WinSmem<64>::kTotal);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWThreads2, WinSmem<64>::kTotal, s>>>(
        p, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
        const_cast<void*>(tree), q_start, n_q, (float*)part);
  }
  return cudaGetLastError();
}

}  // namespace recsa
