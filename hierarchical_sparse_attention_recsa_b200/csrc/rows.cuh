// Row-access helpers shared by the cluster decode and the warp prefill kernels.
//
// A row of d values is spread over d/8 lanes; each lane holds four rotate-half
// pairs (j0..j0+3 and j0+d/2..j0+d/2+3), so RoPE rotation is local to the lane
// and every load is a 16-byte (fp32) or 8-byte (bf16) vector.
#pragma once

#include "recsa_internal.cuh"

namespace recsa {

__device__ __forceinline__ unsigned order_key(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Four rotate-half pairs (j0..j0+3, and the same + d/2) of one row, as fp32.
template <typename T, int HALF>
struct PairLoad;
template <int HALF>
struct PairLoad<float, HALF> {
  static __device__ __forceinline__ void load(const float* row, int j0, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + j0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + HALF + j0));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};
template <int HALF>
struct PairLoad<__nv_bfloat16, HALF> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* row, int j0, float* x) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(row + j0));
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(row + HALF + j0));
    float2 f;
    f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.x)); x[0] = f.x; x[1] = f.y;
    f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.y)); x[2] = f.x; x[3] = f.y;
    f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.x)); x[4] = f.x; x[5] = f.y;
    f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.y)); x[6] = f.x; x[7] = f.y;
  }
};

__device__ __forceinline__ void load_cs(const float2* table, int64_t idx, int half, int j0,
                                        float* cs) {
  const float4* p = reinterpret_cast<const float4*>(table + idx * half + j0);
  const float4 a = __ldg(p), b = __ldg(p + 1);
  cs[0] = a.x; cs[1] = a.y; cs[2] = a.z; cs[3] = a.w;
  cs[4] = b.x; cs[5] = b.y; cs[6] = b.z; cs[7] = b.w;
}

// x (4 first-half, 4 second-half values) rotated by the (cos, sin) pairs cs.
__device__ __forceinline__ void rotate8(float* x, const float* cs) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float c = cs[2 * u], s = cs[2 * u + 1];
    const float x1 = x[u], x2 = x[u + 4];
    x[u] = x1 * c - x2 * s;
    x[u + 4] = x2 * c + x1 * s;
  }
}

template <int LPR>
__device__ __forceinline__ float slot_sum(float v) {
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace recsa

namespace recsa {

// Raw bytes of a lane's four pairs: loads of a whole batch are issued before
// any of them is consumed, and converted to fp32 only afterwards, so the
// loads of an unrolled batch overlap in flight.
struct RawPairs {
  uint4 a, b;
};

template <typename T, int HALF>
struct RawLoad;
template <int HALF>
struct RawLoad<float, HALF> {
  static __device__ __forceinline__ void load(const float* row, int j0, RawPairs& r) {
    r.a = __ldg(reinterpret_cast<const uint4*>(row + j0));
    r.b = __ldg(reinterpret_cast<const uint4*>(row + HALF + j0));
  }
  static __device__ __forceinline__ void cvt(const RawPairs& r, float* x) {
    x[0] = __uint_as_float(r.a.x); x[1] = __uint_as_float(r.a.y);
    x[2] = __uint_as_float(r.a.z); x[3] = __uint_as_float(r.a.w);
    x[4] = __uint_as_float(r.b.x); x[5] = __uint_as_float(r.b.y);
    x[6] = __uint_as_float(r.b.z); x[7] = __uint_as_float(r.b.w);
  }
};
template <int HALF>
struct RawLoad<__nv_bfloat16, HALF> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* row, int j0, RawPairs& r) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(row + j0));
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(row + HALF + j0));
    r.a.x = a.x; r.a.y = a.y;
    r.b.x = b.x; r.b.y = b.y;
  }
  static __device__ __forceinline__ float lo(unsigned u) { return __uint_as_float(u << 16); }
  static __device__ __forceinline__ float hi(unsigned u) { return __uint_as_float(u & 0xffff0000u); }
  static __device__ __forceinline__ void cvt(const RawPairs& r, float* x) {
    x[0] = lo(r.a.x); x[1] = hi(r.a.x); x[2] = lo(r.a.y); x[3] = hi(r.a.y);
    x[4] = lo(r.b.x); x[5] = hi(r.b.x); x[6] = lo(r.b.y); x[7] = hi(r.b.y);
  }
};

}  // namespace recsa

namespace recsa {

// Raw bytes of a lane's four pairs of a bf16 row (half the registers of
// RawPairs); loaded first, converted after the whole batch is in flight.
struct RawBf {
  uint2 a, b;
};
template <int HALF>
__device__ __forceinline__ void raw_load_bf(const __nv_bfloat16* row, int j0, RawBf& r) {
  r.a = __ldg(reinterpret_cast<const uint2*>(row + j0));
  r.b = __ldg(reinterpret_cast<const uint2*>(row + HALF + j0));
}
__device__ __forceinline__ void raw_cvt_bf(const RawBf& r, float* x) {
  x[0] = __uint_as_float(r.a.x << 16); x[1] = __uint_as_float(r.a.x & 0xffff0000u);
  x[2] = __uint_as_float(r.a.y << 16); x[3] = __uint_as_float(r.a.y & 0xffff0000u);
  x[4] = __uint_as_float(r.b.x << 16); x[5] = __uint_as_float(r.b.x & 0xffff0000u);
  x[6] = __uint_as_float(r.b.y << 16); x[7] = __uint_as_float(r.b.y & 0xffff0000u);
}
// Token-row loader for either dtype: bf16 rows use RawBf, fp32 rows RawPairs.
template <typename T, int HALF>
struct TokRow {
  RawPairs r;
  __device__ __forceinline__ void zero() {
    r.a = make_uint4(0u, 0u, 0u, 0u);
    r.b = make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ void load(const T* row, int j0) { RawLoad<T, HALF>::load(row, j0, r); }
  __device__ __forceinline__ void cvt(float* x) const { RawLoad<T, HALF>::cvt(r, x); }
};
template <int HALF>
struct TokRow<__nv_bfloat16, HALF> {
  RawBf r;
  __device__ __forceinline__ void zero() {
    r.a = make_uint2(0u, 0u);
    r.b = make_uint2(0u, 0u);
  }
  __device__ __forceinline__ void load(const __nv_bfloat16* row, int j0) {
    raw_load_bf<HALF>(row, j0, r);
  }
  __device__ __forceinline__ void cvt(float* x) const { raw_cvt_bf(r, x); }
};

}  // namespace recsa

namespace recsa {

// Asynchronous 16-byte global -> shared copies (no registers held while in
// flight); wait with cp_async_wait_all() and a barrier before reading.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gsrc));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// A lane's four pairs of a row held in shared memory (dtype T), as fp32.
template <typename T, int HALF>
struct SharedPairs;
template <int HALF>
struct SharedPairs<__nv_bfloat16, HALF> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* row, int j0, float* x) {
    RawBf r;
    r.a = *reinterpret_cast<const uint2*>(row + j0);
    r.b = *reinterpret_cast<const uint2*>(row + HALF + j0);
    raw_cvt_bf(r, x);
  }
};
template <int HALF>
struct SharedPairs<float, HALF> {
  static __device__ __forceinline__ void load(const float* row, int j0, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(row + j0);
    const float4 b = *reinterpret_cast<const float4*>(row + HALF + j0);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// (cos, sin) pairs advanced by a fixed rotation: cs <- cs * step (per pair,
// as complex numbers), for rows whose RoPE index grows by a constant stride.
__device__ __forceinline__ void advance_cs(float* cs, const float* step) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float c = cs[2 * u], s = cs[2 * u + 1];
    cs[2 * u] = c * step[2 * u] - s * step[2 * u + 1];
    cs[2 * u + 1] = s * step[2 * u] + c * step[2 * u + 1];
  }
}

}  // namespace recsa

namespace recsa {

// Bulk prefetch of a contiguous global range into L2 by the TMA unit (one
// instruction per range; 16-byte aligned address, size a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

}  // namespace recsa

namespace recsa {

// One online-softmax fold of score s with value pairs v.
__device__ __forceinline__ void fold8(float& m, float& l, float* acc, float s, const float* v) {
  if (s > m) {
    const float r = __expf(m - s);
    l = l * r + 1.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = fmaf(acc[c], r, v[c]);
    m = s;
  } else {
    const float w = __expf(s - m);
    l += w;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = fmaf(w, v[c], acc[c]);
  }
}

// Two online-softmax folds (scores s0, s1 with value pairs v0, v1; a row
// that is off is skipped) with one rescale of the state.
__device__ __forceinline__ void fold2(float& m, float& l, float* acc, float s0, bool on0,
                                      const float* v0, float s1, bool on1, const float* v1) {
  s0 = on0 ? s0 : -INFINITY;
  s1 = on1 ? s1 : -INFINITY;
  const float mx = fmaxf(s0, s1);
  if (mx == -INFINITY) return;
  if (mx > m) {
    const float r = __expf(m - mx);
    l *= r;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= r;
    m = mx;
  }
  const float w0 = on0 ? __expf(s0 - m) : 0.f;
  const float w1 = on1 ? __expf(s1 - m) : 0.f;
  l += w0 + w1;
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = fmaf(w0, v0[c], fmaf(w1, v1[c], acc[c]));
}

// A lane's four rotate-half pairs of an fp32 row in shared memory.
__device__ __forceinline__ void lds_pairs(const float* row, int j0, int half, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(row + j0);
  const float4 b = *reinterpret_cast<const float4*>(row + half + j0);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// A lane's four (cos, sin) pairs of a RoPE table row held in shared memory.
__device__ __forceinline__ void lds_cs8(const float* row, int j0, float* cs) {
  const float4 a = *reinterpret_cast<const float4*>(row + 2 * j0);
  const float4 b = *reinterpret_cast<const float4*>(row + 2 * j0 + 4);
  cs[0] = a.x; cs[1] = a.y; cs[2] = a.z; cs[3] = a.w;
  cs[4] = b.x; cs[5] = b.y; cs[6] = b.z; cs[7] = b.w;
}
// out = a * b per (cos, sin) pair, as complex numbers (rotation angles add).
__device__ __forceinline__ void cmul8(float* out, const float* a, const float* b) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    out[2 * u] = a[2 * u] * b[2 * u] - a[2 * u + 1] * b[2 * u + 1];
    out[2 * u + 1] = a[2 * u + 1] * b[2 * u] + a[2 * u] * b[2 * u + 1];
  }
}
// The lane's four rotate-half pairs of x (x[u], x[u + 4]) rotated by the
// angles of cs taken negatively: out = R(-theta) x.
__device__ __forceinline__ void rot_neg8(float* out, const float* x, const float* cs) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float c = cs[2 * u], sn = cs[2 * u + 1];
    const float x1 = x[u], x2 = x[u + 4];
    out[u] = fmaf(x1, c, x2 * sn);
    out[u + 4] = fmaf(x2, c, -x1 * sn);
  }
}
// Partial dot product of a lane's eight values, as two independent chains.
__device__ __forceinline__ float dot8(const float* q, const float* x) {
  float a = q[0] * x[0], b = q[4] * x[4];
#pragma unroll
  for (int c = 1; c < 4; ++c) {
    a = fmaf(q[c], x[c], a);
    b = fmaf(q[4 + c], x[4 + c], b);
  }
  return a + b;
}
// Two slot sums (over the LPR lanes of a row) with interleaved shuffles.
template <int LPR>
__device__ __forceinline__ void slot_sum2(float& a, float& b) {
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) {
    const float ta = __shfl_xor_sync(0xffffffffu, a, o);
    const float tb = __shfl_xor_sync(0xffffffffu, b, o);
    a += ta;
    b += tb;
  }
}

}  // namespace recsa
