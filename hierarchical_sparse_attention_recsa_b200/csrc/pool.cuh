// Node pooling shared by the tree build, the append and the fused decode
// step: one warp pools the children of one node (keys: softmax(r . x / sqrt(d))
// weighted sum; values: mean), each lane owning d/32 contiguous channels.
#pragma once

#include "recsa_internal.cuh"

namespace recsa {

template <typename T, int N>
struct RowIO;

template <>
struct RowIO<float, 4> {
  __device__ static void load(const float* row, int lane, float* x) {
    float4 v = reinterpret_cast<const float4*>(row)[lane];
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ static void store(float* row, int lane, const float* x) {
    reinterpret_cast<float4*>(row)[lane] = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <>
struct RowIO<float, 2> {
  __device__ static void load(const float* row, int lane, float* x) {
    float2 v = reinterpret_cast<const float2*>(row)[lane];
    x[0] = v.x; x[1] = v.y;
  }
  __device__ static void store(float* row, int lane, const float* x) {
    reinterpret_cast<float2*>(row)[lane] = make_float2(x[0], x[1]);
  }
};
template <>
struct RowIO<__nv_bfloat16, 4> {
  __device__ static void load(const __nv_bfloat16* row, int lane, float* x) {
    uint2 u = reinterpret_cast<const uint2*>(row)[lane];
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
  }
};
template <>
struct RowIO<__nv_bfloat16, 2> {
  __device__ static void load(const __nv_bfloat16* row, int lane, float* x) {
    __nv_bfloat162 a = reinterpret_cast<const __nv_bfloat162*>(row)[lane];
    float2 fa = __bfloat1622float2(a);
    x[0] = fa.x; x[1] = fa.y;
  }
};

// One warp pools `n` children into this lane's N channels of key and value:
// keyload(i, x) gives child i's key channels, vbase + i * d its value row.
// Rows are processed in groups of 8 so that eight loads per operand are in
// flight per lane.
template <typename T, int N, typename KeyLoad>
__device__ void pool_children(KeyLoad keyload, const T* vbase, int n, int d, const float* rl,
                              float inv_sqrt_d, int lane, float* key, float* val) {
  float m = -INFINITY, l = 0.f;
  float ak[N], av[N];
#pragma unroll
  for (int c = 0; c < N; ++c) ak[c] = av[c] = 0.f;
  constexpr int U = 8;
  for (int i0 = 0; i0 < n; i0 += U) {
    float kx[U][N], vx[U][N], s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < n) {
        keyload(i0 + u, kx[u]);
        RowIO<T, N>::load(vbase + int64_t(i0 + u) * d, lane, vx[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = 0.f;
      if (i0 + u < n) {
#pragma unroll
        for (int c = 0; c < N; ++c) acc = fmaf(rl[c], kx[u][c], acc);
      }
      s[u] = acc;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) s[u] = warp_sum(s[u]) * inv_sqrt_d;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (i0 + u < n) {
        float mn = fmaxf(m, s[u]);
        float sc = expf(m - mn);
        float w = expf(s[u] - mn);
        l = l * sc + w;
#pragma unroll
        for (int c = 0; c < N; ++c) {
          ak[c] = fmaf(w, kx[u][c], ak[c] * sc);
          av[c] += vx[u][c];
        }
        m = mn;
      }
    }
  }
  float il = 1.f / l, in = 1.f / float(n);
#pragma unroll
  for (int c = 0; c < N; ++c) {
    key[c] = ak[c] * il;
    val[c] = av[c] * in;
  }
}

// pool_children over rows (keys at kbase with row stride ks, default d).
template <typename T, int N>
__device__ void pool_rows(const T* kbase, const T* vbase, int n, int d, const float* rl,
                          float inv_sqrt_d, int lane, float* key, float* val, int64_t ks = 0) {
  if (ks == 0) ks = d;
  pool_children<T, N>(
      [&](int i, float* x) { RowIO<T, N>::load(kbase + int64_t(i) * ks, lane, x); }, vbase, n, d,
      rl, inv_sqrt_d, lane, key, val);
}

// Row format of FP8 key storage: a lane's N contiguous channels as N bytes,
// one fp32 scale = max|key| / 448 per row.
template <int N>
__device__ void store_key_fp8(unsigned char* codes, float* scale, int lane, const float* key) {
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < N; ++c) amax = fmaxf(amax, fabsf(key[c]));
  amax = warp_max(amax);
  const float sc = amax / 448.f;
  unsigned int packed = 0;
#pragma unroll
  for (int c = 0; c < N; ++c)
    packed |= unsigned(sc > 0.f ? float_to_fp8(key[c] / sc) : 0) << (8 * c);
  if constexpr (N == 4)
    reinterpret_cast<unsigned int*>(codes)[lane] = packed;
  else
    reinterpret_cast<unsigned short*>(codes)[lane] = static_cast<unsigned short>(packed);
  if (lane == 0) *scale = sc;
}
template <int N>
__device__ void load_key_fp8(const unsigned char* codes, float scale, int lane, float* x) {
  unsigned int packed;
  if constexpr (N == 4)
    packed = reinterpret_cast<const unsigned int*>(codes)[lane];
  else
    packed = reinterpret_cast<const unsigned short*>(codes)[lane];
#pragma unroll
  for (int c = 0; c < N; ++c) x[c] = fp8_to_float((packed >> (8 * c)) & 0xFFu) * scale;
}

// NVFP4 row format: E2M1 codes, two per byte (lower element in the low
// nibble), one E4M3 scale per 16 elements, one fp32 scale per row.  A lane's
// N contiguous channels are N / 2 bytes; a block of 16 spans 16 / N lanes.
// row scale g = max|key| / (6 * 448); block scale sb = E4M3(block max / (6 g));
// code = E2M1(key / (sb * g)).
template <int N>
__device__ void store_key_nvfp4(unsigned char* codes, unsigned char* bscales, float* rscale,
                                int lane, const float* key) {
  constexpr int LPB = 16 / N;   // lanes per block
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < N; ++c) amax = fmaxf(amax, fabsf(key[c]));
  float bmax = amax;
#pragma unroll
  for (int o = 1; o < LPB; o <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
  amax = warp_max(amax);
  const float g = amax / (6.f * 448.f);
  const unsigned char sbc = g > 0.f ? float_to_fp8(bmax / (6.f * g)) : 0;
  const float den = fp8_to_float(sbc) * g;
  unsigned int packed = 0;
#pragma unroll
  for (int c = 0; c < N; ++c)
    packed |= (den > 0.f ? float_to_fp4(key[c] / den) : 0u) << (4 * c);
  if constexpr (N == 4)
    reinterpret_cast<unsigned short*>(codes)[lane] = static_cast<unsigned short>(packed);
  else
    codes[lane] = static_cast<unsigned char>(packed);
  if (lane % LPB == 0) bscales[lane / LPB] = sbc;
  if (lane == 0) *rscale = g;
}
template <int N>
__device__ void load_key_nvfp4(const unsigned char* codes, const unsigned char* bscales, float g,
                               int lane, float* x) {
  constexpr int LPB = 16 / N;
  unsigned int packed;
  if constexpr (N == 4)
    packed = reinterpret_cast<const unsigned short*>(codes)[lane];
  else
    packed = codes[lane];
  const float den = fp8_to_float(bscales[lane / LPB]) * g;
#pragma unroll
  for (int c = 0; c < N; ++c) x[c] = fp4_to_float(packed >> (4 * c)) * den;
}

template <int N>
__device__ void load_r(const float* r, int lane, float* rl) {
#pragma unroll
  for (int c = 0; c < N; ++c) rl[c] = r[lane * N + c];
}

}  // namespace recsa
