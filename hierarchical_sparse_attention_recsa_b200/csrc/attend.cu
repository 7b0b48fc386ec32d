// Generic RecSA attention kernel (prefill and decode): one CTA per
// (query, sequence, KV head) serves the G query heads that share the KV head.
//
// Per query ("Recursive Sparse Attention: Million-Token Length Extrapolation at
// Logarithmic Cost", abstract):
//   * top-down over the visible levels: candidates = children of the nodes kept
//     one level up, then the orphans (visible nodes whose parent is not
//     visible), in position order; each candidate's logit is
//     <R(c) q, R(i) key> / sqrt(d) with i its index among the c candidates;
//     the top min(k, c) are kept (ties -> lower index), the rest enter the
//     shared softmax with their mean-pooled values;
//   * token level: the kept leaf blocks' tokens then the window [a*B, t],
//     indexed 0..n0-1, query at n0-1, in the same online softmax.
// Scores are one warp per (head, entry) dot product over fp32 rows with the
// rotation folded in; the online-softmax state (max, sum, acc[d]) of each head
// lives in registers of the threads that own its channels.
#include "recsa_internal.cuh"

namespace recsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokChunk = 64;

template <typename T>
__device__ __forceinline__ float ld(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ld<float>(const float* p, int64_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <typename T, int P>  // head_dim = 64 * P
__global__ void __launch_bounds__(kThreads)
attend_kernel(Params p, const T* __restrict__ Q, const T* __restrict__ K,
              const T* __restrict__ V, const void* __restrict__ tree,
              const int64_t* __restrict__ len_dev, int64_t q_start, int n_q, int decode,
              T* __restrict__ O, int32_t* __restrict__ trace, int cmax, int kmax) {
  constexpr int d = 64 * P, half = 32 * P;
  constexpr int U = (8 * d + kThreads - 1) / kThreads;  // channel slots per thread (G <= 8)
  const int G = p.group;
  const int qi = blockIdx.x;
  const int64_t seq = blockIdx.y;
  const int g = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smem[];
  float* qf = reinterpret_cast<float*>(smem);                  // [G][d]
  float* qr = qf + G * d;                                      // [G][d]
  float* score = qr + G * d;                                   // [G][cmax]
  float* wts = score + G * cmax;                               // [G][cmax]
  int* cand = reinterpret_cast<int*>(wts + G * cmax);          // [G][cmax]
  int* rank = cand + G * cmax;                                 // [G][cmax]
  int* kept = rank + G * cmax;                                 // [G][kmax]
  float* tsc = reinterpret_cast<float*>(kept + G * kmax);      // [G][chunk]
  float* tw = tsc + G * kTokChunk;                             // [G][chunk]
  int64_t* tpos = reinterpret_cast<int64_t*>(
      (reinterpret_cast<uintptr_t>(tw + G * kTokChunk) + 7) & ~uintptr_t(7));  // [G][chunk]
  float* mrun = reinterpret_cast<float*>(tpos + G * kTokChunk);  // [G]
  float* lrun = mrun + 8;
  float* scl = lrun + 8;

  const int64_t t = decode ? len_dev[seq] - 1 : q_start + qi;
  const int64_t qrow = ((seq * n_q + qi) * p.hq + int64_t(g) * G) * d;
  const int tstride = kTraceHead + kMaxLevels * p.k;
  if (t < 0 || t >= p.cap) {  // empty sequence, or a length beyond capacity: zeros
    for (int x = tid; x < G * d; x += kThreads) O[qrow + x] = T(0.f);
    return;
  }
  const float2* rope = rope_table(p, tree);
  const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
  const int64_t a = s0 / p.B;
  int64_t vis[kMaxLevels + 2];
  int top = 0;
  {
    int64_t per = 1;
    for (int lev = 1; lev <= p.lay.levels; ++lev) {
      vis[lev] = a / per;
      if (vis[lev] == 0) break;
      top = lev;
      per *= p.b;
    }
  }
  for (int x = tid; x < G * d; x += kThreads) qf[x] = ld<T>(Q, qrow + x);
  if (tid < 8) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }
  float acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.f;
  __syncthreads();

  auto rotate_q = [&](int64_t idx) {
    for (int x = tid; x < G * half; x += kThreads) {
      const int h = x / half, j = x % half;
      const float x1 = qf[h * d + j], x2 = qf[h * d + j + half];
      if (p.rope) {
        const float2 cs = rope[idx * half + j];
        qr[h * d + j] = x1 * cs.x - x2 * cs.y;
        qr[h * d + j + half] = x2 * cs.x + x1 * cs.y;
      } else {
        qr[h * d + j] = x1;
        qr[h * d + j + half] = x2;
      }
    }
  };
  // Dot of head h's rotated query with a row rotated to index idx; warp-wide.
  auto dot_row = [&](int h, const auto* row, int64_t idx) -> float {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < P; ++u) {
      const int j = lane + 32 * u;
      const float k1 = ld(row, j), k2 = ld(row, j + half);
      float r1 = k1, r2 = k2;
      if (p.rope) {
        const float2 cs = rope[idx * half + j];
        r1 = k1 * cs.x - k2 * cs.y;
        r2 = k2 * cs.x + k1 * cs.y;
      }
      s = fmaf(qr[h * d + j], r1, s);
      s = fmaf(qr[h * d + j + half], r2, s);
    }
    return warp_sum(s) * p.inv_sqrt_d;
  };
  // Fold n entries per head (scores in sc[h * ld_] with unselected mask) into
  // the online softmax; rows(h, e) gives the value row.
  auto softmax_update = [&](const float* sc, float* w, int ldw, int n, auto selected,
                            auto vrow) {
    if (warp < G) {
      const int h = warp;
      float mx = -INFINITY;
      for (int e = lane; e < n; e += 32)
        if (!selected(h, e)) mx = fmaxf(mx, sc[h * ldw + e]);
      mx = warp_max(mx);
      if (lane == 0) {
        const float mn = fmaxf(mrun[h], mx);
        scl[h] = (mn == -INFINITY) ? 1.f : expf(mrun[h] - mn);
        mrun[h] = mn;
      }
    }
    __syncthreads();
    for (int x = tid; x < G * n; x += kThreads) {
      const int h = x / n, e = x % n;
      w[h * ldw + e] = selected(h, e) ? 0.f : expf(sc[h * ldw + e] - mrun[h]);
    }
    __syncthreads();
    if (warp < G) {
      const int h = warp;
      float sum = 0.f;
      for (int e = lane; e < n; e += 32) sum += w[h * ldw + e];
      sum = warp_sum(sum);
      if (lane == 0) lrun[h] = lrun[h] * scl[h] + sum;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int x = tid + u * kThreads;
      if (x < G * d) {
        const int h = x / d, c = x % d;
        float a_ = acc[u] * scl[h];
        for (int e = 0; e < n; ++e) {
          const float we = w[h * ldw + e];
          if (we != 0.f) a_ = fmaf(we, ld(vrow(h, e), c), a_);
        }
        acc[u] = a_;
      }
    }
    __syncthreads();
  };

  int kup = 0;
  int64_t ent = 0, keys_read = 0;
  int cnt_c[kMaxLevels + 1], cnt_k[kMaxLevels + 1];
  for (int lev = top; lev >= 1; --lev) {
    const int64_t vup = lev < top ? vis[lev + 1] : 0;
    const int nchild = p.b * kup;
    const int c = nchild + int(vis[lev] - p.b * vup);
    for (int x = tid; x < G * c; x += kThreads) {
      const int h = x / c, ii = x % c;
      cand[h * cmax + ii] = ii < nchild ? kept[h * kmax + ii / p.b] * p.b + ii % p.b
                                        : int(p.b * vup + (ii - nchild));
    }
    rotate_q(c);
    __syncthreads();
    const float* keys = level_keys(p, const_cast<void*>(tree), lev, seq, g);
    const float* vals = level_vals(p, const_cast<void*>(tree), lev, seq, g);
    for (int pr = warp; pr < G * c; pr += kWarps) {
      const int h = pr / c, ii = pr % c;
      const float s = dot_row(h, keys + int64_t(cand[h * cmax + ii]) * d, ii);
      if (lane == 0) score[h * cmax + ii] = s;
    }
    __syncthreads();
    const int kap = c < p.k ? c : p.k;
    for (int x = tid; x < G * c; x += kThreads) {
      const int h = x / c, ii = x % c;
      const float s = score[h * cmax + ii];
      const float* row = score + h * cmax;
      int r = 0;
      for (int jj = 0; jj < c; ++jj) {
        const float sj = row[jj];
        r += (sj > s) || (sj == s && jj < ii);
      }
      rank[h * cmax + ii] = r;
    }
    __syncthreads();
    for (int x = tid; x < G * c; x += kThreads) {
      const int h = x / c, ii = x % c;
      if (rank[h * cmax + ii] < kap) {
        int pos = 0;
        for (int jj = 0; jj < ii; ++jj) pos += rank[h * cmax + jj] < kap;
        kept[h * kmax + pos] = cand[h * cmax + ii];
      }
    }
    __syncthreads();
    softmax_update(
        score, wts, cmax, c, [&](int h, int e) { return rank[h * cmax + e] < kap; },
        [&](int h, int e) { return vals + int64_t(cand[h * cmax + e]) * d; });
    if (trace) {
      for (int x = tid; x < G * kap; x += kThreads) {
        const int h = x / kap, j = x % kap;
        const int64_t rec = ((seq * n_q + qi) * p.hq + int64_t(g) * G + h) * tstride;
        trace[rec + kTraceHead + (lev - 1) * p.k + j] = kept[h * kmax + j];
      }
    }
    cnt_c[lev] = c;
    cnt_k[lev] = kap;
    ent += c - kap;
    keys_read += c;
    kup = kap;
  }

  // Token level: kept leaf blocks, then the window.
  const int nleaf = top > 0 ? kup : 0;
  const int64_t n0 = int64_t(nleaf) * p.B + (t + 1 - a * p.B);
  rotate_q(n0 - 1);
  __syncthreads();
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  for (int64_t base = 0; base < n0; base += kTokChunk) {
    const int nt = int(n0 - base < kTokChunk ? n0 - base : kTokChunk);
    for (int pr = warp; pr < G * nt; pr += kWarps) {
      const int h = pr / nt, tt = pr % nt;
      const int64_t ii = base + tt;
      const int64_t pos = ii < int64_t(nleaf) * p.B
                              ? int64_t(kept[h * kmax + ii / p.B]) * p.B + ii % p.B
                              : a * p.B + (ii - int64_t(nleaf) * p.B);
      const float s = dot_row(h, K + (kvbase + pos) * d, ii);
      if (lane == 0) {
        tsc[h * kTokChunk + tt] = s;
        tpos[h * kTokChunk + tt] = pos;
      }
    }
    __syncthreads();
    softmax_update(
        tsc, tw, kTokChunk, nt, [&](int, int) { return false; },
        [&](int h, int e) { return V + (kvbase + tpos[h * kTokChunk + e]) * d; });
  }
  ent += n0;
  keys_read += n0;

#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int x = tid + u * kThreads;
    if (x < G * d) {
      const int h = x / d;
      const float o = acc[u] / lrun[h];
      if constexpr (sizeof(T) == 2)
        O[qrow + x] = __float2bfloat16_rn(o);
      else
        O[qrow + x] = o;
    }
  }
  if (trace && tid < G) {
    const int64_t rec = ((seq * n_q + qi) * p.hq + int64_t(g) * G + tid) * tstride;
    trace[rec + 0] = top;
    trace[rec + 1] = int32_t(ent);
    trace[rec + 2] = int32_t(keys_read);
    trace[rec + 3] = int32_t(n0);
    for (int lev = 1; lev <= kMaxLevels; ++lev) {
      const bool on = lev <= top;
      trace[rec + 4 + lev - 1] = on ? cnt_c[lev] : 0;
      trace[rec + 4 + kMaxLevels + lev - 1] = on ? cnt_k[lev] : 0;
    }
  }
}

template <typename T, int P>
cudaError_t attend_typed(const Params& p, const void* Q, const void* K, const void* V,
                         const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                         int decode, void* O, int32_t* trace, cudaStream_t s) {
  const int d = 64 * P;
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  int64_t cm = p.b * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  const int cmax = int(cm < 1 ? 1 : cm);
  const int kmax = int(kk < cmax ? kk : cmax);
  const int G = p.group;
  size_t bytes = size_t(G) * d * 4 * 2 + size_t(G) * cmax * 16 + size_t(G) * kmax * 4 +
                 size_t(G) * kTokChunk * 8 + 8 + size_t(G) * kTokChunk * 8 + 3 * 8 * 4 + 64;
  if (bytes > 200 * 1024) return cudaErrorInvalidConfiguration;
  auto kern = attend_kernel<T, P>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(bytes));
  if (e != cudaSuccess) return e;
  if (p.batch > 65535 || p.hkv > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid(n_q, p.batch, p.hkv);
  kern<<<grid, kThreads, bytes, s>>>(p, reinterpret_cast<const T*>(Q),
                                     reinterpret_cast<const T*>(K), reinterpret_cast<const T*>(V),
                                     tree, len_dev, q_start, n_q, decode, reinterpret_cast<T*>(O),
                                     trace, cmax, kmax);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const Params& p, const void* Q, const void* K, const void* V,
                          const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                          int decode, void* O, int32_t* trace, cudaStream_t s) {
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? attend_typed<__nv_bfloat16, 2>(p, Q, K, V, tree, len_dev, q_start, n_q,
                                                       decode, O, trace, s)
                      : attend_typed<__nv_bfloat16, 1>(p, Q, K, V, tree, len_dev, q_start, n_q,
                                                       decode, O, trace, s);
  return p.d == 128 ? attend_typed<float, 2>(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O,
                                             trace, s)
                    : attend_typed<float, 1>(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O,
                                             trace, s);
}

}  // namespace recsa
