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
//
// The same kernel serves the selection variants of the geometry's mode:
//   * RECSA_MODE_GROUP: the G heads' scores give one group score per candidate
//     (the sum of the heads' softmax probabilities over the level's
//     candidates), ranked once and shared by the heads;
//   * RECSA_MODE_ZHA ("Subquadratic Attention with a Hierarchical
//     Tree-Structured Indexer", Figure 3 caption): un-rotated routing scores
//     (the best of a node's reference keys, decoded from FP8 or NVFP4 when the
//     keys are stored so), a per-head top-p set capped at k, no summaries in
//     the softmax, and the reached leaves plus the window at true positions.
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
template <>   // FP8 E4M3 key codes
__device__ __forceinline__ float ld<unsigned char>(const unsigned char* p, int64_t i) {
  return fp8_to_float(p[i]);
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
  // ZHA: per-head routed counts (the expanded node count differs per head)
  int* zkup = reinterpret_cast<int*>(scl + 8);                 // [8] expanded one level up
  int* zc = zkup + 8;                                          // [8][kMaxLevels + 1] candidates
  int* zk = zc + 8 * (kMaxLevels + 1);                         // [8][kMaxLevels + 1] expanded
  // GROUP: per head max and sum of exp over the level's candidates
  float* gmx = reinterpret_cast<float*>(zk + 8 * (kMaxLevels + 1));   // [8]
  float* gsm = gmx + 8;                                               // [8]

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
  if (tid < 8) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; zkup[tid] = 0; }
  float acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.f;
  __syncthreads();

  const bool zha = p.mode == RECSA_MODE_ZHA;
  const bool group = p.mode == RECSA_MODE_GROUP;
  constexpr int LS = kMaxLevels + 1;
  // Query rotated to index idx (idx < 0: copied un-rotated).
  auto rotate_q = [&](int64_t idx) {
    for (int x = tid; x < G * half; x += kThreads) {
      const int h = x / half, j = x % half;
      const float x1 = qf[h * d + j], x2 = qf[h * d + j + half];
      if (p.rope && idx >= 0) {
        const float2 cs = rope[idx * half + j];
        qr[h * d + j] = x1 * cs.x - x2 * cs.y;
        qr[h * d + j + half] = x2 * cs.x + x1 * cs.y;
      } else {
        qr[h * d + j] = x1;
        qr[h * d + j + half] = x2;
      }
    }
  };
  // Dot of head h's rotated query with a row rotated to index idx (idx < 0:
  // not rotated); warp-wide.
  auto dot_row = [&](int h, const auto* row, int64_t idx) -> float {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < P; ++u) {
      const int j = lane + 32 * u;
      const float k1 = ld(row, j), k2 = ld(row, j + half);
      float r1 = k1, r2 = k2;
      if (p.rope && idx >= 0) {
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

  // Per head: expanded count one level up (zkup), candidates and kept per
  // level (zc, zk).  Under RecSA every head has the same counts; under ZHA
  // the top-p set size, hence the next level's candidates, differ per head.
  for (int lev = top; lev >= 1; --lev) {
    const int64_t vup = lev < top ? vis[lev + 1] : 0;
    const int norph = int(vis[lev] - p.b * vup);
    int cmx = 0;
    for (int h = 0; h < G; ++h) cmx = max(cmx, p.b * zkup[h] + norph);
    for (int x = tid; x < G * cmx; x += kThreads) {
      const int h = x / cmx, ii = x % cmx;
      const int nchild = p.b * zkup[h];
      if (ii < nchild + norph)
        cand[h * cmax + ii] = ii < nchild ? kept[h * kmax + ii / p.b] * p.b + ii % p.b
                                          : int(p.b * vup + (ii - nchild));
    }
    // RecSA: candidate-local positions, query at index c (all heads share c).
    // ZHA: plain dot products of the un-rotated query and summary keys.
    rotate_q(zha ? -1 : cmx);
    __syncthreads();
    const float* keys = level_keys(p, const_cast<void*>(tree), lev, seq, g);
    const float* vals = level_vals(p, const_cast<void*>(tree), lev, seq, g);
    for (int pr = warp; pr < G * cmx; pr += kWarps) {
      const int h = pr / cmx, ii = pr % cmx;
      if (ii >= p.b * zkup[h] + norph) continue;  // warp-uniform
      // a node with several reference keys (ZHA) scores its best match
      const int64_t node = cand[h * cmax + ii];
      float s;
      if (p.kfmt == RECSA_KEYS_FP8) {   // codes times the row's scale
        const unsigned char* kc = level_kcodes(p, const_cast<void*>(tree), lev, seq, g) +
                                  node * p.nref * d;
        const float* ks = level_kscales(p, const_cast<void*>(tree), lev, seq, g) + node * p.nref;
        s = dot_row(h, kc, -1) * ks[0];
        for (int ref = 1; ref < p.nref; ++ref) s = fmaxf(s, dot_row(h, kc + ref * d, -1) * ks[ref]);
      } else if (p.kfmt == RECSA_KEYS_NVFP4) {   // E2M1 codes x block scale, x row scale
        const unsigned char* kc = level_kcodes(p, const_cast<void*>(tree), lev, seq, g) +
                                  node * p.nref * p.kcb;
        const unsigned char* kb = level_kbscales(p, const_cast<void*>(tree), lev, seq, g) +
                                  node * p.nref * (d / 16);
        const float* ks = level_kscales(p, const_cast<void*>(tree), lev, seq, g) + node * p.nref;
        s = -INFINITY;
        for (int ref = 0; ref < p.nref; ++ref) {
          const unsigned char* c0 = kc + ref * p.kcb;
          const unsigned char* b0 = kb + ref * (d / 16);
          float acc_ = 0.f;
#pragma unroll
          for (int u = 0; u < P; ++u) {
            const int j = lane + 32 * u;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int e = j + hf * half;
              const float v = fp4_to_float(c0[e >> 1] >> (4 * (e & 1))) * fp8_to_float(b0[e >> 4]);
              acc_ = fmaf(qr[h * d + e], v, acc_);
            }
          }
          s = fmaxf(s, warp_sum(acc_) * p.inv_sqrt_d * ks[ref]);
        }
      } else {
        const float* kr = keys + node * p.nref * d;
        s = dot_row(h, kr, zha ? -1 : ii);
        for (int ref = 1; ref < p.nref; ++ref) s = fmaxf(s, dot_row(h, kr + ref * d, -1));
      }
      if (lane == 0) score[h * cmax + ii] = s;
    }
    __syncthreads();
    if (group) {
      // One selection for the G heads (all have c = cmx candidates): group
      // score = sum over heads of the candidate's softmax probability, ranked
      // with ties to the lower index; every head gets the shared ranks.
      if (warp < G) {
        const float* row = score + warp * cmax;
        float mx = -INFINITY;
        for (int e = lane; e < cmx; e += 32) mx = fmaxf(mx, row[e]);
        mx = warp_max(mx);
        float sm = 0.f;
        for (int e = lane; e < cmx; e += 32) sm += expf(row[e] - mx);
        sm = warp_sum(sm);
        if (lane == 0) {
          gmx[warp] = mx;
          gsm[warp] = sm;
        }
      }
      __syncthreads();
      for (int ii = tid; ii < cmx; ii += kThreads) {
        float agg = 0.f;
        for (int h = 0; h < G; ++h) agg += expf(score[h * cmax + ii] - gmx[h]) / gsm[h];
        wts[ii] = agg;
      }
      __syncthreads();
      for (int ii = tid; ii < cmx; ii += kThreads) {
        const float s = wts[ii];
        int r = 0;
        for (int jj = 0; jj < cmx; ++jj) {
          const float sj = wts[jj];
          r += (sj > s) || (sj == s && jj < ii);
        }
        for (int h = 0; h < G; ++h) rank[h * cmax + ii] = r;
      }
    }
    for (int x = tid; x < G * cmx && !group; x += kThreads) {
      const int h = x / cmx, ii = x % cmx;
      const int c = p.b * zkup[h] + norph;
      if (ii >= c) continue;
      const float s = score[h * cmax + ii];
      const float* row = score + h * cmax;
      int r = 0;
      for (int jj = 0; jj < c; ++jj) {
        const float sj = row[jj];
        r += (sj > s) || (sj == s && jj < ii);
      }
      rank[h * cmax + ii] = r;
      if (zha && r == 0) scl[h] = s;  // the level's maximum score
    }
    __syncthreads();
    if (zha) {
      // Top-p: weights exp(s - max) laid out in rank order, then the shortest
      // rank prefix whose mass reaches p of the total, capped at min(k, c).
      for (int x = tid; x < G * cmx; x += kThreads) {
        const int h = x / cmx, ii = x % cmx;
        if (ii < p.b * zkup[h] + norph)
          wts[h * cmax + rank[h * cmax + ii]] = expf(score[h * cmax + ii] - scl[h]);
      }
      __syncthreads();
      if (warp < G) {
        const int h = warp;
        const int c = p.b * zkup[h] + norph;
        const int cap = c < p.k ? c : p.k;
        int cnt = cap;
        if (p.top_p < 1.f) {
          float tot = 0.f;
          for (int e = lane; e < c; e += 32) tot += wts[h * cmax + e];
          const float thr = p.top_p * warp_sum(tot);
          float run = 0.f;
          for (int b0 = 0; b0 < c; b0 += 32) {
            const int e = b0 + lane;
            float x = e < c ? wts[h * cmax + e] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const float y = __shfl_up_sync(0xffffffffu, x, o);
              if (lane >= o) x += y;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, e < c && run + x >= thr);
            if (hit) {
              cnt = min(cnt, b0 + __ffs(hit));
              break;
            }
            run += __shfl_sync(0xffffffffu, x, 31);
          }
        }
        if (lane == 0) {
          zc[h * LS + lev] = c;
          zk[h * LS + lev] = cnt;
        }
      }
    } else if (tid < G) {
      const int c = p.b * zkup[tid] + norph;
      zc[tid * LS + lev] = c;
      zk[tid * LS + lev] = c < p.k ? c : p.k;
    }
    __syncthreads();
    for (int x = tid; x < G * cmx; x += kThreads) {
      const int h = x / cmx, ii = x % cmx;
      const int kap = zk[h * LS + lev];
      if (ii < zc[h * LS + lev] && rank[h * cmax + ii] < kap) {
        int pos = 0;
        for (int jj = 0; jj < ii; ++jj) pos += rank[h * cmax + jj] < kap;
        kept[h * kmax + pos] = cand[h * cmax + ii];
      }
    }
    __syncthreads();
    if (!zha)  // RecSA: unselected summaries join the softmax
      softmax_update(
          score, wts, cmax, cmx,
          [&](int h, int e) { return rank[h * cmax + e] < zk[h * LS + lev]; },
          [&](int h, int e) { return vals + int64_t(cand[h * cmax + e]) * d; });
    if (trace) {
      for (int x = tid; x < G * kmax; x += kThreads) {
        const int h = x / kmax, j = x % kmax;
        if (j >= zk[h * LS + lev]) continue;
        const int64_t rec = ((seq * n_q + qi) * p.hq + int64_t(g) * G + h) * tstride;
        trace[rec + kTraceHead + (lev - 1) * p.k + j] = kept[h * kmax + j];
      }
    }
    if (tid < G) zkup[tid] = zk[tid * LS + lev];
    __syncthreads();
  }

  // Token level: kept leaf blocks, then the window.  RecSA indexes them
  // 0..n0-1 with the query at n0-1; ZHA keeps their true positions.
  auto n0_of = [&](int h) -> int64_t {
    return int64_t(top > 0 ? zkup[h] : 0) * p.B + (t + 1 - a * p.B);
  };
  int64_t n0max = 0;
  for (int h = 0; h < G; ++h) n0max = n0_of(h) > n0max ? n0_of(h) : n0max;
  rotate_q(zha ? t : n0max - 1);
  __syncthreads();
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  for (int64_t base = 0; base < n0max; base += kTokChunk) {
    const int nt = int(n0max - base < kTokChunk ? n0max - base : kTokChunk);
    for (int pr = warp; pr < G * nt; pr += kWarps) {
      const int h = pr / nt, tt = pr % nt;
      const int64_t ii = base + tt;
      if (ii >= n0_of(h)) continue;  // warp-uniform
      const int64_t nleaf = top > 0 ? zkup[h] : 0;
      const int64_t pos = ii < nleaf * p.B ? int64_t(kept[h * kmax + ii / p.B]) * p.B + ii % p.B
                                           : a * p.B + (ii - nleaf * p.B);
      const float s = dot_row(h, K + (kvbase + pos) * d, zha ? pos : ii);
      if (lane == 0) {
        tsc[h * kTokChunk + tt] = s;
        tpos[h * kTokChunk + tt] = pos;
      }
    }
    __syncthreads();
    softmax_update(
        tsc, tw, kTokChunk, nt, [&](int h, int e) { return base + e >= n0_of(h); },
        [&](int h, int e) { return V + (kvbase + tpos[h * kTokChunk + e]) * d; });
  }

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
    const int64_t n0 = n0_of(tid);
    int64_t ent = n0, keys_read = n0;
    for (int lev = 1; lev <= top; ++lev) {
      keys_read += zc[tid * LS + lev];
      if (!zha) ent += zc[tid * LS + lev] - zk[tid * LS + lev];
    }
    trace[rec + 0] = top;
    trace[rec + 1] = int32_t(ent);
    trace[rec + 2] = int32_t(keys_read);
    trace[rec + 3] = int32_t(n0);
    for (int lev = 1; lev <= kMaxLevels; ++lev) {
      const bool on = lev <= top;
      trace[rec + 4 + lev - 1] = on ? zc[tid * LS + lev] : 0;
      trace[rec + 4 + kMaxLevels + lev - 1] = on ? zk[tid * LS + lev] : 0;
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
                 size_t(G) * kTokChunk * 8 + 8 + size_t(G) * kTokChunk * 8 + 3 * 8 * 4 + 64 +
                 size_t(8 + 16 * (kMaxLevels + 1) + 16) * 4;
  if (bytes > 200 * 1024) return cudaErrorInvalidConfiguration;
  auto kern = attend_kernel<T, P>;
  cudaError_t e = ensure_smem(kern, int(bytes));
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
