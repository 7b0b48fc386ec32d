// Prefill, exact local window on tensor cores.
//
// For a query at t the window is the token range [a*B, t] (a = floor(max(0,
// t+1-W)/B)).  Its tokens are indexed after the kept leaves' tokens and the
// query sits at the last index, so the RoPE angle between query and window
// token is t - pos, the true distance ("Recursive Sparse Attention:
// Million-Token Length Extrapolation at Logarithmic Cost", abstract:
// candidate-local positions; the token level's window keeps its order).  The
// window is therefore a banded causal attention that consecutive queries
// share: a CTA takes 64 query rows (64/G consecutive queries x the G heads of
// one KV group) and streams the union of their windows in chunks of 64 keys.
//
// Keys and queries are rotated to a CTA-local origin (the first query's
// window start) in fp32, rounded to fp16 (10-bit mantissa) and multiplied
// with mma.sync m16n8k16 (fp32 accumulation): S = Q K^T, masked to each row's
// band, online softmax in registers (FlashAttention-2 register reuse of S as
// the A operand of P V), then O = P V.  The result is this window's partial
// softmax: per (query, head) a row of the caller workspace receives the
// normalised output, the max and the sum in fp32; the tree kernel folds the
// summaries and kept leaves into it and writes O once.  ZHA routing attends
// the same window at true positions ("Subquadratic Attention with a
// Hierarchical Tree-Structured Indexer", Figure 3 caption), so its prefill
// takes the same partials and its routing kernel merges the reached leaves
// into them.  Work per CTA is ~20 MFLOP against ~0.3 MB of K/V reads, so the
// kernel is far from both rooflines; the tree part of the prefill dominates.
#include <cuda_fp16.h>

#include "recsa_internal.cuh"

namespace recsa {
namespace {

constexpr int kRows = 64;          // query rows (query x head) per CTA
constexpr int kChunk = 64;         // keys per chunk
constexpr int kWThreads = 128;     // 4 warps x 16 rows

__device__ __forceinline__ unsigned pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const unsigned*>(&h);
}

__device__ __forceinline__ void mma16816(float* c, const unsigned* a, unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kWThreads, 3)
window_mma_kernel(Params p, const __nv_bfloat16* __restrict__ Q,
                  const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                  const void* __restrict__ tree, int64_t q_start, int n_q,
                  float* __restrict__ part) {
  constexpr int HALF = D / 2, QP = D + 8, VP = kChunk + 8;
  const int G = p.group, QB = kRows / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int64_t seq = blockIdx.y / p.hkv;
  const int g = int(blockIdx.y % p.hkv);
  const int q0 = blockIdx.x * QB;                       // first query index of the CTA
  const int nqh = min(QB, n_q - q0);
  const int64_t t0 = q_start + q0;
  const int64_t tl = t0 + nqh - 1;
  auto win_lo = [&](int64_t t) -> int64_t {
    const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
    return s0 / p.B * p.B;
  };
  const int64_t base = win_lo(t0);                      // CTA-local RoPE origin
  const int64_t kend = tl + 1;

  extern __shared__ __align__(16) unsigned char smem[];
  __half* Qs = reinterpret_cast<__half*>(smem);         // [kRows][QP]
  __half* Ks = Qs + kRows * QP;                         // [kChunk][QP]
  __half* Vt = Ks + kChunk * QP;                        // [D][VP]
  int* lo_q = reinterpret_cast<int*>(Vt + D * VP);      // [QB] window start - base

  const float2* rope = rope_table(p, tree);
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;

  for (int qq = tid; qq < QB; qq += kWThreads)
    lo_q[qq] = qq < nqh ? int(win_lo(t0 + qq) - base) : 1 << 30;
  // Q rows rotated by (t - base)
  for (int x = tid; x < kRows * HALF; x += kWThreads) {
    const int row = x / HALF, j = x % HALF;
    const int qq = row / G, h = row % G;
    float y1 = 0.f, y2 = 0.f;
    if (qq < nqh) {
      const int64_t qi = q0 + qq;
      const __nv_bfloat16* q = Q + ((seq * n_q + qi) * p.hq + int64_t(g) * G + h) * D;
      const float x1 = __bfloat162float(q[j]), x2 = __bfloat162float(q[j + HALF]);
      if (p.rope) {
        const float2 cs = rope[(t0 + qq - base) * HALF + j];
        y1 = x1 * cs.x - x2 * cs.y;
        y2 = x2 * cs.x + x1 * cs.y;
      } else {
        y1 = x1;
        y2 = x2;
      }
    }
    Qs[row * QP + j] = __float2half_rn(y1);
    Qs[row * QP + j + HALF] = __float2half_rn(y2);
  }
  __syncthreads();

  // A fragments of this warp's 16 rows for every 16-wide k step (kept in registers).
  const int r0 = warp * 16;
  unsigned qa[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int c = kk * 16 + tig * 2;
    qa[kk][0] = *reinterpret_cast<const unsigned*>(Qs + (r0 + gid) * QP + c);
    qa[kk][1] = *reinterpret_cast<const unsigned*>(Qs + (r0 + gid + 8) * QP + c);
    qa[kk][2] = *reinterpret_cast<const unsigned*>(Qs + (r0 + gid) * QP + c + 8);
    qa[kk][3] = *reinterpret_cast<const unsigned*>(Qs + (r0 + gid + 8) * QP + c + 8);
  }
  // Band limits of this thread's two rows (relative to base).
  const int rowA = r0 + gid, rowB = r0 + gid + 8;
  const int qqA = rowA / G, qqB = rowB / G;
  const int loA = lo_q[qqA], loB = lo_q[qqB];
  const int hiA = qqA < nqh ? int(t0 + qqA - base) : -1;
  const int hiB = qqB < nqh ? int(t0 + qqB - base) : -1;

  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
  float oacc[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
  const float scale = p.inv_sqrt_d;

  for (int64_t kb = base; kb < kend; kb += kChunk) {
    __syncthreads();
    // stage the chunk: K rotated by (pos - base), V transposed, both fp16
    for (int x = tid; x < kChunk * HALF; x += kWThreads) {
      const int key = x / HALF, j = x % HALF;
      const int64_t pos = kb + key;
      float y1 = 0.f, y2 = 0.f;
      if (pos < kend) {
        const __nv_bfloat16* k = K + (kvbase + pos) * D;
        const float x1 = __bfloat162float(k[j]), x2 = __bfloat162float(k[j + HALF]);
        if (p.rope) {
          const float2 cs = rope[(pos - base) * HALF + j];
          y1 = x1 * cs.x - x2 * cs.y;
          y2 = x2 * cs.x + x1 * cs.y;
        } else {
          y1 = x1;
          y2 = x2;
        }
      }
      Ks[key * QP + j] = __float2half_rn(y1);
      Ks[key * QP + j + HALF] = __float2half_rn(y2);
    }
    for (int x = tid; x < kChunk * D; x += kWThreads) {
      const int key = x / D, dim = x % D;
      const int64_t pos = kb + key;
      const float v = pos < kend ? __bfloat162float(V[(kvbase + pos) * D + dim]) : 0.f;
      Vt[dim * VP + key] = __float2half_rn(v);
    }
    __syncthreads();

    // S = Q K^T for 16 rows x 64 keys
    float s[kChunk / 8][4];
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; ++nt) {
        const __half* kr = Ks + (nt * 8 + gid) * QP + kk * 16 + tig * 2;
        mma16816(s[nt], qa[kk], *reinterpret_cast<const unsigned*>(kr),
                 *reinterpret_cast<const unsigned*>(kr + 8));
      }
    }
    // mask to each row's band, online softmax
    const int kr0 = int(kb - base);
    float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = kr0 + nt * 8 + tig * 2 + e;
        s[nt][e] = (key >= loA && key <= hiA) ? s[nt][e] * scale : -INFINITY;
        s[nt][2 + e] = (key >= loB && key <= hiB) ? s[nt][2 + e] * scale : -INFINITY;
        mxA = fmaxf(mxA, s[nt][e]);
        mxB = fmaxf(mxB, s[nt][2 + e]);
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, o));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, o));
    }
    const float mnA = fmaxf(mA, mxA), mnB = fmaxf(mB, mxB);
    const float rA = (mnA == -INFINITY) ? 1.f : __expf(mA - mnA);
    const float rB = (mnB == -INFINITY) ? 1.f : __expf(mB - mnB);
    float sumA = 0.f, sumB = 0.f;
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[nt][e] = (s[nt][e] == -INFINITY) ? 0.f : __expf(s[nt][e] - mnA);
        s[nt][2 + e] = (s[nt][2 + e] == -INFINITY) ? 0.f : __expf(s[nt][2 + e] - mnB);
        sumA += s[nt][e];
        sumB += s[nt][2 + e];
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      sumA += __shfl_xor_sync(0xffffffffu, sumA, o);
      sumB += __shfl_xor_sync(0xffffffffu, sumB, o);
    }
    lA = lA * rA + sumA;
    lB = lB * rB + sumB;
    mA = mnA;
    mB = mnB;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      oacc[nt][0] *= rA;
      oacc[nt][1] *= rA;
      oacc[nt][2] *= rB;
      oacc[nt][3] *= rB;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kChunk / 16; ++kk) {
      unsigned pa[4];
      pa[0] = pack_half2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_half2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_half2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_half2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const __half* vr = Vt + (nt * 8 + gid) * VP + kk * 16 + tig * 2;
        mma16816(oacc[nt], pa, *reinterpret_cast<const unsigned*>(vr),
                 *reinterpret_cast<const unsigned*>(vr + 8));
      }
    }
  }

  // partial row per (query, head), fp32: normalised window output [D], max, sum
  const int hA = rowA % G, hB = rowB % G;
  const float iA = lA > 0.f ? 1.f / lA : 0.f, iB = lB > 0.f ? 1.f / lB : 0.f;
  if (qqA < nqh) {
    float* row = part + ((seq * n_q + q0 + qqA) * p.hq + int64_t(g) * G + hA) * (D + 2);
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *reinterpret_cast<float2*>(row + nt * 8 + tig * 2) =
          make_float2(oacc[nt][0] * iA, oacc[nt][1] * iA);
    if (tig == 0) *reinterpret_cast<float2*>(row + D) = make_float2(mA, lA);
  }
  if (qqB < nqh) {
    float* row = part + ((seq * n_q + q0 + qqB) * p.hq + int64_t(g) * G + hB) * (D + 2);
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *reinterpret_cast<float2*>(row + nt * 8 + tig * 2) =
          make_float2(oacc[nt][2] * iB, oacc[nt][3] * iB);
    if (tig == 0) *reinterpret_cast<float2*>(row + D) = make_float2(mB, lB);
  }
}

}  // namespace

// Window partials for a prefill range; cudaErrorNotSupported when the
// geometry is outside this kernel's limits (bf16 only; the RoPE table must
// reach W + B + 64/G indices).
cudaError_t launch_prefill_window(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, int64_t q_start, int32_t n_q, void* part,
                                  cudaStream_t s) {
  // the tcgen05 kernel first (RECSA_PREFILL_PATH = 1 keeps this mma.sync one)
  if (switches().prefill_path != 1) {
    const cudaError_t e = launch_prefill_window_tc(p, Q, K, V, tree, q_start, n_q, part, s);
    if (e != cudaErrorNotSupported) return e;
    cudaGetLastError();
  }
  // the window is attended at true distances t - pos: the same for RecSA and
  // ZHA (group selection attends it in the generic kernel)
  if (p.mode != RECSA_MODE_RECSA && p.mode != RECSA_MODE_ZHA) return cudaErrorNotSupported;
  if (p.dtype != RECSA_DTYPE_BF16) return cudaErrorNotSupported;
  if (p.group < 1 || kRows % p.group) return cudaErrorNotSupported;
  const int QB = kRows / p.group;
  if (p.rope && int64_t(p.W) + p.B + QB > p.lay.rope_rows) return cudaErrorNotSupported;
  if (int64_t(p.batch) * p.hkv > 65535) return cudaErrorNotSupported;
  const int D = p.d;
  const size_t bytes = size_t(kRows + kChunk) * (D + 8) * 2 + size_t(D) * (kChunk + 8) * 2 +
                       size_t(QB) * 4 + 16;
  dim3 grid(unsigned((n_q + QB - 1) / QB), unsigned(p.batch * p.hkv));
  cudaError_t e;
  if (D == 128) {
    auto kern = window_mma_kernel<128>;
    e = ensure_smem(kern, int(bytes));
    if (e != cudaSuccess) return e;
    kern<<<grid, kWThreads, bytes, s>>>(p, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                        (const __nv_bfloat16*)V, tree, q_start, n_q,
                                        (float*)part);
  } else {
    auto kern = window_mma_kernel<64>;
    e = ensure_smem(kern, int(bytes));
    if (e != cudaSuccess) return e;
    kern<<<grid, kWThreads, bytes, s>>>(p, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                        (const __nv_bfloat16*)V, tree, q_start, n_q,
                                        (float*)part);
  }
  return cudaGetLastError();
}

}  // namespace recsa
