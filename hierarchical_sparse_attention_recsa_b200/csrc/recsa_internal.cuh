// Internal definitions shared by the RecSA CUDA translation units: the tree
// buffer layout, the launch parameter block and small device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/recsa.h"

namespace recsa {

constexpr int kMaxLevels = RECSA_MAX_LEVELS;
constexpr int kHeaderBytes = 256;
constexpr int kTraceHead = 4 + 2 * kMaxLevels;  // ints before the kept-id lists
// Per-sequence step counters of the fused decode step live in the tree header.
constexpr int kStepCounterOffset = 64;
constexpr int kStepCounters = (kHeaderBytes - kStepCounterOffset) / 4;

// Byte layout of the caller-owned tree buffer (computed on the host).
struct TreeLayout {
  int32_t levels;                 // summary levels at capacity (D)
  int32_t rope_rows;              // rows of the RoPE table
  int64_t nodes[kMaxLevels];      // nodes per (sequence, KV head) at level l+1
  int64_t key_off[kMaxLevels];    // fp32 keys  [batch][Hkv][nodes][nref][d]
  int64_t val_off[kMaxLevels];    // fp32 values [batch][Hkv][nodes][d]
  int64_t kscale_off[kMaxLevels]; // FP8 / NVFP4 keys: fp32 row scales [batch][Hkv][nodes][nref]
  int64_t kbscale_off[kMaxLevels];// NVFP4 keys: E4M3 block scales [..][nref][d / 16]
  int64_t rope_off;               // float2 (cos, sin) [rope_rows][d/2]
  int64_t total;
};

// Everything a kernel needs about the geometry, passed by value.
struct Params {
  int32_t dtype, d, hq, hkv, group, B, b, k, W, rope, batch;
  int32_t Bsh, bsh;   // log2 of B and b when powers of two, else -1
  int32_t mode;       // RECSA_MODE_RECSA or RECSA_MODE_ZHA
  float top_p;        // ZHA routing mass
  int32_t nref;       // reference queries per pooler (keys per node), >= 1
  int32_t kfmt;       // RECSA_KEYS_F32, RECSA_KEYS_FP8 or RECSA_KEYS_NVFP4
  int32_t kcb;        // code bytes per key row (FP8: d, NVFP4: d / 2)
  int32_t test_expire;   // decode: one extra wait nothing completes (bounded-wait tests)
  int64_t cap;
  float inv_sqrt_d;
  TreeLayout lay;
};

// x / B, x % B, x / b, x % b for non-negative 32-bit x (shifts when powers of two).
__device__ __forceinline__ int div_B(const Params& p, int x) { return p.Bsh >= 0 ? x >> p.Bsh : x / p.B; }
__device__ __forceinline__ int mod_B(const Params& p, int x) { return p.Bsh >= 0 ? x & (p.B - 1) : x % p.B; }
__device__ __forceinline__ int div_b(const Params& p, int x) { return p.bsh >= 0 ? x >> p.bsh : x / p.b; }
__device__ __forceinline__ int mod_b(const Params& p, int x) { return p.bsh >= 0 ? x & (p.b - 1) : x % p.b; }

// Device error word at offset 0 of the tree header.
__device__ __forceinline__ unsigned int* tree_error_word(void* tree) {
  return reinterpret_cast<unsigned int*>(tree);
}

__device__ __forceinline__ float* level_keys(const Params& p, void* tree, int lev /*1-based*/,
                                             int64_t seq, int g) {
  char* base = reinterpret_cast<char*>(tree) + p.lay.key_off[lev - 1];
  return reinterpret_cast<float*>(base) + ((seq * p.hkv + g) * p.lay.nodes[lev - 1]) * p.nref * p.d;
}
// Low-precision key storage: codes [nodes][nref][kcb] bytes, (NVFP4) block
// scales [nodes][nref][d / 16] bytes, row scales [nodes][nref] fp32.
__device__ __forceinline__ unsigned char* level_kcodes(const Params& p, void* tree, int lev,
                                                       int64_t seq, int g) {
  char* base = reinterpret_cast<char*>(tree) + p.lay.key_off[lev - 1];
  return reinterpret_cast<unsigned char*>(base) +
         ((seq * p.hkv + g) * p.lay.nodes[lev - 1]) * p.nref * p.kcb;
}
__device__ __forceinline__ unsigned char* level_kbscales(const Params& p, void* tree, int lev,
                                                         int64_t seq, int g) {
  char* base = reinterpret_cast<char*>(tree) + p.lay.kbscale_off[lev - 1];
  return reinterpret_cast<unsigned char*>(base) +
         ((seq * p.hkv + g) * p.lay.nodes[lev - 1]) * p.nref * (p.d / 16);
}
__device__ __forceinline__ float* level_kscales(const Params& p, void* tree, int lev, int64_t seq,
                                                int g) {
  char* base = reinterpret_cast<char*>(tree) + p.lay.kscale_off[lev - 1];
  return reinterpret_cast<float*>(base) + ((seq * p.hkv + g) * p.lay.nodes[lev - 1]) * p.nref;
}
__device__ __forceinline__ float* level_vals(const Params& p, void* tree, int lev, int64_t seq,
                                             int g) {
  char* base = reinterpret_cast<char*>(tree) + p.lay.val_off[lev - 1];
  return reinterpret_cast<float*>(base) + ((seq * p.hkv + g) * p.lay.nodes[lev - 1]) * p.d;
}
__device__ __forceinline__ const float2* rope_table(const Params& p, const void* tree) {
  return reinterpret_cast<const float2*>(reinterpret_cast<const char*>(tree) + p.lay.rope_off);
}

// FP8 E4M3 code <-> float with CUDA's conversions (nearest, ties to even,
// saturated at +-448).
__device__ __forceinline__ float fp8_to_float(unsigned char c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return float(v);
}
__device__ __forceinline__ unsigned char float_to_fp8(float x) {
  return __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
// FP4 E2M1 code (low nibble) <-> float, CUDA's conversions (nearest, ties to
// even, saturated at +-6).
__device__ __forceinline__ float fp4_to_float(unsigned int c) {
  return __half2float(__half(__nv_cvt_fp4_to_halfraw(__nv_fp4_storage_t(c & 0xFu), __NV_E2M1)));
}
__device__ __forceinline__ unsigned int float_to_fp4(float x) {
  return unsigned(__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest)) & 0xFu;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Element load from a K/V/Q tensor of the geometry's dtype, as fp32.
__device__ __forceinline__ float load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == RECSA_DTYPE_BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}
__device__ __forceinline__ void store_elem(void* base, int64_t idx, float v, int dtype) {
  if (dtype == RECSA_DTYPE_BF16)
    reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(base)[idx] = v;
}

// Kernel-variant switches taken from the environment (RECSA_ZHA_GENERIC,
// RECSA_DECODE_GENERIC, RECSA_PREFILL_GENERIC, RECSA_DECODE_SPLIT="hpc,s",
// RECSA_PREFILL_PATH, RECSA_TEST_EXPIRE_WAIT).  They are read once, on the
// first call into the library, and again only by recsa_reload_switches(), so
// no launch pays for getenv().
struct Switches {
  int zha_generic, decode_generic, prefill_generic, test_expire;
  int split_hpc, split_s;   // forced decode launch shape; 0 = automatic
  int prefill_path;         // forced prefill path (0 = automatic); see recsa_api.cu
};
const Switches& switches();
void reload_switches();

// Raise `func`'s dynamic shared memory limit on the current device to at
// least `bytes`, calling cudaFuncSetAttribute only when the limit recorded for
// this (kernel, device) is lower: launches then cost no attribute call.
cudaError_t ensure_smem(const void* func, int bytes);
template <typename F>
cudaError_t ensure_smem(F* func, int bytes) {
  return ensure_smem(reinterpret_cast<const void*>(func), bytes);
}
// cudaFuncAttributeNonPortableClusterSizeAllowed = 1, once per (kernel, device).
cudaError_t ensure_nonportable_cluster(const void* func);
template <typename F>
cudaError_t ensure_nonportable_cluster(F* func) {
  return ensure_nonportable_cluster(reinterpret_cast<const void*>(func));
}

// Host-side launchers (defined in the .cu files).
cudaError_t launch_rope_table(const Params& p, void* tree, double rope_base, cudaStream_t s);
cudaError_t launch_build(const Params& p, const void* K, const void* V, const int64_t* len_host,
                         const float* r, int64_t r_stride, void* tree, cudaStream_t s);
cudaError_t launch_append(const Params& p, void* K, void* V, const void* k_new, const void* v_new,
                          int64_t* len_dev, const float* r, int64_t r_stride, void* tree,
                          cudaStream_t s);
cudaError_t launch_attend(const Params& p, const void* Q, const void* K, const void* V,
                          const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                          int decode, void* O, int32_t* trace, cudaStream_t s);
// Cluster decode kernel; cudaErrorNotSupported when the geometry is outside its limits.
// ZHA routing variant (mode RECSA_MODE_ZHA): one CTA per (query, sequence,
// query head); a prefill given the window kernel's partials (wpart) merges
// them instead of attending the window.  cudaErrorNotSupported outside its
// limits.
cudaError_t launch_zha(const Params& p, const void* Q, const void* K, const void* V,
                       const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                       int decode, void* O, int32_t* trace, const void* wpart, cudaStream_t s);
cudaError_t launch_decode_cluster(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                                  int32_t* trace, cudaStream_t s);
// Fused decode step: append (token write, pooling of completed nodes, length
// update) and decode in one cluster launch; cudaErrorNotSupported when the
// geometry or batch is outside its limits.
cudaError_t launch_decode_step(const Params& p, const void* Q, void* K, void* V,
                               const void* k_new, const void* v_new, int64_t* len_dev,
                               const float* r, int64_t r_stride, void* tree, int32_t n_q,
                               void* O, int32_t* trace, cudaStream_t s);
// Warp-per-(query, head) prefill kernel; cudaErrorNotSupported outside its limits.
// wpart: window partials from launch_prefill_window (fp32 rows of d + 2 per
// (sequence, query, head): normalised output, max, sum), or null to let this
// kernel attend the window itself.
cudaError_t launch_prefill_warp(const Params& p, const void* Q, const void* K, const void* V,
                                const void* tree, int64_t q_start, int32_t n_q, void* O,
                                int32_t* trace, const void* wpart, cudaStream_t s);
// Output of the prefill traversal when the kept leaves are attended by the
// tensor-core leaf path (prefill_leaf.cu) instead of by the traversal itself.
struct LeafOut {
  float* part;    // [rows][d + 2]: partial softmax (normalised output, max, sum) of
                  // the window and the unselected summaries; may alias the window partials
  int2* kept;     // [rows][kmax]: {leaf bucket, position in that bucket's pair list}
  int* nkept;     // [rows]: kept leaves of the query head
  int* counts;    // [batch * n_kv_heads * nleaf]: pairs per leaf bucket (zeroed first)
  int nleaf;      // level-1 nodes per (sequence, KV head) at capacity
  int kmax;       // kept-leaf slots per query head
};
// The traversal of launch_prefill_warp writing a LeafOut instead of O.
cudaError_t launch_prefill_warp_leafout(const Params& p, const void* Q, const void* K,
                                        const void* V, const void* tree, int64_t q_start,
                                        int32_t n_q, int32_t* trace, const void* wpart,
                                        const LeafOut& lo, cudaStream_t s);
// The tree levels of a prefill as tensor-core tiles grouped by parent node
// (prefill_tree.cu): lo.part holds the window partial on entry and the window
// + summaries partial on return; the kept leaves go to lo.kept/nkept/counts.
bool prefill_tree_supported(const Params& p);
size_t prefill_tree_workspace_need(const Params& p, int32_t n_q);
cudaError_t launch_prefill_tree(const Params& p, const void* Q, const void* tree,
                                int64_t q_start, int32_t n_q, int32_t* trace, const LeafOut& lo,
                                void* ws, cudaStream_t s);
// Prefill with the kept leaves on the tensor cores (prefill_leaf.cu): the
// workspace holds every intermediate (prefill_tc_workspace_need bytes).
bool prefill_tc_supported(const Params& p);
size_t prefill_tc_workspace_need(const Params& p, int32_t n_q);
cudaError_t launch_prefill_tc(const Params& p, const void* Q, const void* K, const void* V,
                              const void* tree, int64_t q_start, int32_t n_q, void* O,
                              int32_t* trace, void* ws, cudaStream_t s);
// Prefill with the window partials kept in a fixed device array (no caller
// workspace) of prefill_static_bytes() bytes.
cudaError_t launch_prefill_static(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, int64_t q_start, int32_t n_q, void* O,
                                  int32_t* trace, cudaStream_t s);
size_t prefill_static_bytes();
// Bytes of window partials for n_q queries per sequence (fp32 rows of d + 2).
size_t prefill_workspace_need(const Params& p, int32_t n_q);
// The same window partials from the tcgen05 window kernel (window_tc.cu).
cudaError_t launch_prefill_window_tc(const Params& p, const void* Q, const void* K,
                                     const void* V, const void* tree, int64_t q_start,
                                     int32_t n_q, void* part, cudaStream_t s);
// Tensor-core window partials for a prefill range (bf16) into part (fp32
// rows of d + 2); cudaErrorNotSupported outside its limits.
cudaError_t launch_prefill_window(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, int64_t q_start, int32_t n_q, void* part,
                                  cudaStream_t s);

}  // namespace recsa
