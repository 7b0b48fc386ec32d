// Prefill attention: one warp per (query, head); a CTA's eight warps serve two
// consecutive queries of one KV group, so their window and upper-level rows
// are shared through L1.
//
// Per query ("Recursive Sparse Attention: Million-Token Length Extrapolation at
// Logarithmic Cost", abstract): the window tokens and the top level are scored
// in the first pass; every later pass scores one level's candidates while
// folding the previous level's unselected summaries into the online softmax;
// the last pass folds level 1's unselected summaries and the kept leaves'
// tokens.  Selection is a warp top-k (redux.sync on order-preserving keys,
// ties to the lower index).  Rows are read into registers with vector loads,
// d/8 lanes per row, four rotate-half pairs per lane.  No block-level
// barriers: every warp runs independently, so many queries are in flight per
// SM to cover the dependent gathers.
#include "recsa_internal.cuh"
#include "rows.cuh"

namespace recsa {
namespace {

constexpr int kPThreads = 256;
constexpr int kPWarps = kPThreads / 32;
constexpr int kPRegSlots = 8;   // top-k candidates held in registers: 32 per slot

enum PItem { pKey = 0, pVal = 1, pNone = 2 };

template <typename T, int D>
__global__ void __launch_bounds__(kPThreads, 3)
prefill_warp_kernel(Params p, const T* __restrict__ Q, const T* __restrict__ K,
                    const T* __restrict__ V, const void* __restrict__ tree, int64_t q_start,
                    int n_q, T* __restrict__ O, int32_t* __restrict__ trace, int cmax, int kmax,
                    int warp_bytes, const float* wpart, LeafOut lo) {
  constexpr int HALF = D / 2, LPR = HALF / 4, SPW = 32 / LPR;
  const int G = p.group;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPR, slot = lane / LPR, j0 = 4 * sub;
  const int64_t item = int64_t(blockIdx.x) * kPWarps + warp;
  const int64_t seq = blockIdx.y / p.hkv;
  const int g = int(blockIdx.y % p.hkv);
  if (item >= int64_t(n_q) * G) return;   // whole warp exits; no block barriers follow
  const int qi = int(item / G);
  const int h = g * G + int(item % G);
  const int64_t t = q_start + qi;

  extern __shared__ __align__(16) unsigned char smem[];
  float* qf = reinterpret_cast<float*>(smem + size_t(warp) * warp_bytes);
  float* qlev = qf + D;
  float* qtok = qlev + D;
  float* sc = qtok + D;                                          // [2][cmax]
  int* kept = reinterpret_cast<int*>(sc + 2 * cmax);             // [2][kmax]
  unsigned char* kfl = reinterpret_cast<unsigned char*>(kept + 2 * kmax);  // [2][cmax]

  const float2* rope = rope_table(p, tree);
  const int rmax = p.lay.rope_rows - 1;
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
  int cnt_c[kMaxLevels + 2], cnt_k[kMaxLevels + 2];
  {
    int kup = 0;
    for (int lev = top; lev >= 1; --lev) {
      const int64_t vup = lev < top ? vis[lev + 1] : 0;
      cnt_c[lev] = p.b * kup + int(vis[lev] - p.b * vup);
      cnt_k[lev] = cnt_c[lev] < p.k ? cnt_c[lev] : p.k;
      kup = cnt_k[lev];
    }
  }
  const int nleaf = top > 0 ? cnt_k[1] : 0;
  const int64_t n_win = t + 1 - a * p.B;
  const int64_t n0 = int64_t(nleaf) * p.B + n_win;
  const int64_t qrow = ((seq * n_q + qi) * p.hq + h) * D;
  for (int x = lane; x < D; x += 32) qf[x] = load_elem(Q, qrow + x, p.dtype);
  __syncwarp();
  auto rotate_q = [&](float* dst, int64_t idx) {
    for (int j = lane; j < HALF; j += 32) {
      const float x1 = qf[j], x2 = qf[j + HALF];
      if (p.rope) {
        const float2 cs = rope[idx * HALF + j];
        dst[j] = x1 * cs.x - x2 * cs.y;
        dst[j + HALF] = x2 * cs.x + x1 * cs.y;
      } else {
        dst[j] = x1;
        dst[j + HALF] = x2;
      }
    }
    __syncwarp();
  };
  rotate_q(qtok, n0 - 1);

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;

  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  const float inv_sqrt_d = p.inv_sqrt_d;
  const int tstride = kTraceHead + kMaxLevels * p.k;
  const int64_t rec = ((seq * n_q + qi) * p.hq + h) * int64_t(tstride);

  auto cand_node = [&](int lev, int i) -> int {
    const int kup = lev < top ? cnt_k[lev + 1] : 0;
    const int vup = lev < top ? int(vis[lev + 1]) : 0;
    if (i < p.b * kup) return kept[((lev + 1) & 1) * kmax + div_b(p, i)] * p.b + mod_b(p, i);
    return p.b * vup + (i - p.b * kup);
  };

  // Token rows: the window [a*B, t] (when this kernel attends it) or the
  // kept leaves' tokens, each at its token-level index; K/V rows in dtype,
  // two rows per lane slot at a time.  The score of a row at index i is
  // <R(n0 - 1) q, R(i) k> = <R(n0 - 1 - i) q, k>: the query (rotated to
  // n0 - 1 in qtok) is turned back by the row's index instead of rotating
  // the key; a slot's rows advance by SPW, so its query turns by R(-SPW).
  auto token_loop = [&](bool window) {
    const int nt = window ? int(n_win) : nleaf * p.B;
    const int win0 = int(a) * p.B;
    const int idx0 = window ? nleaf * p.B : 0;
    const int* kept1 = kept + 1 * kmax;                           // level 1 = parity 1
    float q0[8], st[8], st2[8];
    lds_pairs(qtok, j0, HALF, q0);
    if (p.rope) {
      float cs[8], t2[8];
      load_cs(rope, min(idx0 + slot, rmax), HALF, j0, cs);
      load_cs(rope, min(SPW, rmax), HALF, j0, st);
      rot_neg8(t2, q0, cs);
#pragma unroll
      for (int c = 0; c < 8; ++c) q0[c] = t2[c];
      cmul8(st2, st, st);
    }
    for (int base = 0; base < nt; base += 2 * SPW) {
      const int e0 = base + slot, e1 = e0 + SPW;
      const bool on0 = e0 < nt, on1 = e1 < nt;
      TokRow<T, HALF> rk0, rv0, rk1, rv1;
      rk0.zero(); rv0.zero(); rk1.zero(); rv1.zero();
      if (on0) {
        const int pos = window ? win0 + e0 : kept1[div_B(p, e0)] * p.B + mod_B(p, e0);
        rk0.load(K + (kvbase + pos) * D, j0);
        rv0.load(V + (kvbase + pos) * D, j0);
      }
      if (on1) {
        const int pos = window ? win0 + e1 : kept1[div_B(p, e1)] * p.B + mod_B(p, e1);
        rk1.load(K + (kvbase + pos) * D, j0);
        rv1.load(V + (kvbase + pos) * D, j0);
      }
      float k0[8], v0[8], k1[8], v1[8], q1[8];
      rk0.cvt(k0);
      rv0.cvt(v0);
      rk1.cvt(k1);
      rv1.cvt(v1);
      if (p.rope) {
        rot_neg8(q1, q0, st);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) q1[c] = q0[c];
      }
      float s0 = dot8(q0, k0), s1 = dot8(q1, k1);
      if (p.rope) {
        float t2[8];
        rot_neg8(t2, q0, st2);
#pragma unroll
        for (int c = 0; c < 8; ++c) q0[c] = t2[c];
      }
      slot_sum2<LPR>(s0, s1);
      fold2(m, l, acc, s0 * inv_sqrt_d, on0, v0, s1 * inv_sqrt_d, on1, v1);
    }
  };

  // Tree rows, two items per lane slot at a time: key candidates of level
  // klev (scored into sc; candidate i sits at item i, and the query in qlev
  // is turned back by i as for the tokens) and the unselected candidates of
  // level vlev (values folded); fp32 rows.
  auto tree_loop = [&](int klev, int vlev) {
    const int nk = klev > 0 ? cnt_c[klev] : 0;
    const int nv = vlev > 0 ? cnt_c[vlev] : 0;
    const int total = nk + nv;
    const float* keys = klev > 0 ? level_keys(p, const_cast<void*>(tree), klev, seq, g) : nullptr;
    const float* vals = vlev > 0 ? level_vals(p, const_cast<void*>(tree), vlev, seq, g) : nullptr;
    const int kupK = (klev > 0 && klev < top) ? cnt_k[klev + 1] : 0;
    const int nchK = p.b * kupK;
    const int orphK = (klev > 0 && klev < top) ? p.b * int(vis[klev + 1]) - nchK : 0;
    const int* keptK = kept + ((klev + 1) & 1) * kmax;
    const int kupV = (vlev > 0 && vlev < top) ? cnt_k[vlev + 1] : 0;
    const int nchV = p.b * kupV;
    const int orphV = (vlev > 0 && vlev < top) ? p.b * int(vis[vlev + 1]) - nchV : 0;
    const int* keptV = kept + ((vlev + 1) & 1) * kmax;
    const float* scV = sc + (vlev & 1) * cmax;
    const unsigned char* flV = kfl + (vlev & 1) * cmax;
    float* scK = sc + (klev & 1) * cmax;
    float q0[8], st[8], st2[8];
    lds_pairs(qlev, j0, HALF, q0);
    if (p.rope) {
      float cs[8], t2[8];
      load_cs(rope, min(slot, rmax), HALF, j0, cs);
      load_cs(rope, min(SPW, rmax), HALF, j0, st);
      rot_neg8(t2, q0, cs);
#pragma unroll
      for (int c = 0; c < 8; ++c) q0[c] = t2[c];
      cmul8(st2, st, st);
    }
    for (int base = 0; base < total; base += 2 * SPW) {
      RawPairs ra[2];
      int kind[2], idx[2];
      float sv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = base + u * SPW + slot;
        kind[u] = pNone;
        idx[u] = 0;
        sv[u] = 0.f;
        ra[u].a = make_uint4(0u, 0u, 0u, 0u);
        ra[u].b = make_uint4(0u, 0u, 0u, 0u);
        if (e < nk) {
          const int i = e;
          const int node = i < nchK ? keptK[div_b(p, i)] * p.b + mod_b(p, i) : orphK + i;
          kind[u] = pKey;
          idx[u] = i;
          RawLoad<float, HALF>::load(keys + int64_t(node) * D, j0, ra[u]);
        } else if (e < total) {
          const int i = e - nk;
          if (!flV[i]) {
            const int node = i < nchV ? keptV[div_b(p, i)] * p.b + mod_b(p, i) : orphV + i;
            kind[u] = pVal;
            sv[u] = scV[i];
            RawLoad<float, HALF>::load(vals + int64_t(node) * D, j0, ra[u]);
          }
        }
      }
      float x0[8], x1[8], q1[8];
      RawLoad<float, HALF>::cvt(ra[0], x0);
      RawLoad<float, HALF>::cvt(ra[1], x1);
      if (p.rope) {
        rot_neg8(q1, q0, st);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) q1[c] = q0[c];
      }
      float s0 = dot8(q0, x0), s1 = dot8(q1, x1);
      if (p.rope) {
        float t2[8];
        rot_neg8(t2, q0, st2);
#pragma unroll
        for (int c = 0; c < 8; ++c) q0[c] = t2[c];
      }
      if (__any_sync(0xffffffffu, kind[0] == pKey || kind[1] == pKey)) slot_sum2<LPR>(s0, s1);
      if (kind[0] == pKey) {
        if (sub == 0) scK[idx[0]] = s0 * inv_sqrt_d;
      } else if (kind[0] == pVal) {
        fold8(m, l, acc, sv[0], x0);
      }
      if (kind[1] == pKey) {
        if (sub == 0) scK[idx[1]] = s1 * inv_sqrt_d;
      } else if (kind[1] == pVal) {
        fold8(m, l, acc, sv[1], x1);
      }
    }
  };

  auto run_pass = [&](bool window, int klev, int vlev, bool tokens) {
    if (window) token_loop(true);
    if (klev > 0 || vlev > 0) tree_loop(klev, vlev);
    if (tokens) token_loop(false);
    __syncwarp();
  };

  // Warp top-k: kap rounds of an arg-max over order-preserving keys held in
  // registers (lane l holds candidates l, l + 32, ...; 0 = none or taken);
  // redux.sync gives the round's maximum, a ballot its lanes, and on a tie of
  // keys the lowest index wins.  Candidates beyond 32 * kPRegSlots are read
  // from shared memory in the same rounds.  The kept list is compacted in
  // index order with one ballot per row of 32 candidates.
  auto topk = [&](int lev) {
    const int c = cnt_c[lev], kap = cnt_k[lev];
    const int par = lev & 1;
    const float* scl = sc + par * cmax;
    unsigned char* fl = kfl + par * cmax;
    int* kp = kept + par * kmax;
    const int ns = (c + 31) >> 5;
    unsigned taken = 0;
    if (kap >= c) {
      for (int s = 0; s < ns; ++s)
        if (s * 32 + lane < c) taken |= 1u << s;
    } else {
      unsigned key[kPRegSlots];
#pragma unroll
      for (int s = 0; s < kPRegSlots; ++s) {
        const int i = s * 32 + lane;
        key[s] = i < c ? order_key(scl[i]) : 0u;
      }
      for (int r = 0; r < kap; ++r) {
        unsigned bk = key[0];
        int bs = 0;
#pragma unroll
        for (int s = 1; s < kPRegSlots; ++s)
          if (key[s] > bk) {
            bk = key[s];
            bs = s;
          }
        for (int s = kPRegSlots; s < ns; ++s) {
          const int i = s * 32 + lane;
          if (i < c && !((taken >> s) & 1u)) {
            const unsigned kk = order_key(scl[i]);
            if (kk > bk) {
              bk = kk;
              bs = s;
            }
          }
        }
        const unsigned M = __reduce_max_sync(0xffffffffu, bk);
        unsigned who = __ballot_sync(0xffffffffu, bk == M);
        if (__popc(who) > 1) {
          const unsigned I =
              __reduce_min_sync(0xffffffffu, bk == M ? unsigned(bs * 32 + lane) : 0xffffffffu);
          who = 1u << (I & 31u);
        }
        if ((who >> lane) & 1u) {
          taken |= 1u << bs;
#pragma unroll
          for (int s = 0; s < kPRegSlots; ++s)
            if (s == bs) key[s] = 0u;
        }
      }
    }
    int cnt = 0;
    for (int s = 0; s < ns; ++s) {
      const int i = s * 32 + lane;
      const bool f = i < c && ((taken >> s) & 1u);
      if (i < c) fl[i] = f;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (f) {
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        const int node = cand_node(lev, i);
        kp[pos] = node;
        if (trace) trace[rec + kTraceHead + (lev - 1) * p.k + pos] = node;
      }
      cnt += __popc(bal);
    }
    __syncwarp();
  };

  // With window partials from the tensor-core window kernel (wpart != null)
  // the window rows are skipped here and merged at the end.
  const bool own_window = wpart == nullptr;
  if (top > 0) {
    rotate_q(qlev, cnt_c[top]);
    run_pass(own_window, top, 0, false);
    topk(top);
    for (int lev = top - 1; lev >= 1; --lev) {
      rotate_q(qlev, cnt_c[lev]);
      run_pass(false, lev, lev + 1, false);
      topk(lev);
    }
    if (lo.counts) {
      // kept leaves are attended by the tensor-core leaf path: list them and
      // take each pair's position in its leaf's pair list
      const int64_t qh_row = (seq * n_q + qi) * p.hq + h;
      const int* kept1 = kept + 1 * kmax;
      for (int s = lane; s < nleaf; s += 32) {
        const int64_t bucket = (seq * p.hkv + g) * int64_t(lo.nleaf) + kept1[s];
        const int pos = atomicAdd(lo.counts + bucket, 1);
        lo.kept[qh_row * lo.kmax + s] = make_int2(int(bucket), pos);
      }
    }
    run_pass(false, 0, 1, lo.counts == nullptr);
  } else if (own_window) {
    run_pass(true, 0, 0, false);
  }

  // merge the lane slots, write O
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o);
    const float lo = __shfl_xor_sync(0xffffffffu, l, o);
    const float mn = fmaxf(m, mo);
    const float ra_ = (m == -INFINITY) ? 0.f : __expf(m - mn);
    const float rb_ = (mo == -INFINITY) ? 0.f : __expf(mo - mn);
    l = l * ra_ + lo * rb_;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[c], o);
      acc[c] = acc[c] * ra_ + ao * rb_;
    }
    m = mn;
  }
  if (lo.counts) {
    // partial softmax of the window and the summaries (normalised output, max, sum)
    const int64_t qh_row = (seq * n_q + qi) * p.hq + h;
    float mm = m, ra_ = 1.f, rb_ = 0.f;
    float o1[4], o2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) o1[c] = o2[c] = 0.f;
    if (!own_window) {
      const float* wrow = wpart + qh_row * (D + 2);
      const float2 w = *reinterpret_cast<const float2*>(wrow + D);
      mm = fmaxf(m, w.x);
      ra_ = (m == -INFINITY) ? 0.f : __expf(m - mm);
      rb_ = (w.x == -INFINITY) ? 0.f : __expf(w.x - mm) * w.y;
      if (lane < LPR) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          o1[c] = wrow[j0 + c];
          o2[c] = wrow[HALF + j0 + c];
        }
      }
    }
    const float lsum = l * ra_ + rb_;
    const float il = 1.f / lsum;
    // every lane has read its window values before any lane overwrites the row
    __syncwarp();
    if (lane < LPR) {
      float* prow = lo.part + qh_row * (D + 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        prow[j0 + c] = (acc[c] * ra_ + o1[c] * rb_) * il;
        prow[HALF + j0 + c] = (acc[4 + c] * ra_ + o2[c] * rb_) * il;
      }
      if (lane == 0) *reinterpret_cast<float2*>(prow + D) = make_float2(mm, lsum);
    }
    if (lane == 0) lo.nkept[qh_row] = nleaf;
  } else if (lane < LPR) {
    if (own_window) {
      const float il = 1.f / l;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        store_elem(O, qrow + j0 + c, acc[c] * il, p.dtype);
        store_elem(O, qrow + HALF + j0 + c, acc[4 + c] * il, p.dtype);
      }
    } else {
      // merge with the window's partial softmax (normalised output, max, sum)
      const float* wrow = wpart + ((seq * n_q + qi) * p.hq + h) * (D + 2);
      const float2 w = *reinterpret_cast<const float2*>(wrow + D);
      const float mm = fmaxf(m, w.x);
      const float ra_ = (m == -INFINITY) ? 0.f : __expf(m - mm);
      const float rb_ = (w.x == -INFINITY) ? 0.f : __expf(w.x - mm) * w.y;
      const float il = 1.f / (l * ra_ + rb_);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float o1 = wrow[j0 + c];
        const float o2 = wrow[HALF + j0 + c];
        store_elem(O, qrow + j0 + c, (acc[c] * ra_ + o1 * rb_) * il, p.dtype);
        store_elem(O, qrow + HALF + j0 + c, (acc[4 + c] * ra_ + o2 * rb_) * il, p.dtype);
      }
    }
  }
  if (trace && lane == 0) {
    int64_t e = 0, r = 0;
    for (int lev = 1; lev <= top; ++lev) {
      e += cnt_c[lev] - cnt_k[lev];
      r += cnt_c[lev];
    }
    trace[rec + 0] = top;
    trace[rec + 1] = int32_t(e + n0);
    trace[rec + 2] = int32_t(r + n0);
    trace[rec + 3] = int32_t(n0);
    for (int lev = 1; lev <= kMaxLevels; ++lev) {
      trace[rec + 4 + lev - 1] = lev <= top ? cnt_c[lev] : 0;
      trace[rec + 4 + kMaxLevels + lev - 1] = lev <= top ? cnt_k[lev] : 0;
    }
  }
}

template <typename T, int D>
cudaError_t prefill_typed(const Params& p, const void* Q, const void* K, const void* V,
                          const void* tree, int64_t q_start, int32_t n_q, void* O, int32_t* trace,
                          const void* wpart, const LeafOut& lo, cudaStream_t s) {
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  int64_t cm = p.b * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  const int cmax = int(cm < 1 ? 1 : cm);
  const int kmax = int(kk < cmax ? kk : cmax);
  if (cmax > 1024) return cudaErrorNotSupported;
  const int warp_bytes = int(((3 * D + 2 * cmax) * 4 + 2 * kmax * 4 + 2 * cmax + 15) / 16 * 16);
  const size_t bytes = size_t(warp_bytes) * kPWarps;
  if (bytes > 200 * 1024) return cudaErrorNotSupported;
  auto kern = prefill_warp_kernel<T, D>;
  cudaError_t e = ensure_smem(kern, int(bytes));
  if (e != cudaSuccess) return e;
  const int64_t items = int64_t(n_q) * p.group;
  const int64_t blocks = (items + kPWarps - 1) / kPWarps;
  if (blocks > 0x7fffffff || int64_t(p.batch) * p.hkv > 65535) return cudaErrorNotSupported;
  dim3 grid(unsigned(blocks), unsigned(p.batch * p.hkv));
  kern<<<grid, kPThreads, bytes, s>>>(p, reinterpret_cast<const T*>(Q),
                                      reinterpret_cast<const T*>(K),
                                      reinterpret_cast<const T*>(V), tree, q_start, n_q,
                                      reinterpret_cast<T*>(O), trace, cmax, kmax, warp_bytes,
                                      reinterpret_cast<const float*>(wpart), lo);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_warp(const Params& p, const void* Q, const void* K, const void* V,
                                const void* tree, int64_t q_start, int32_t n_q, void* O,
                                int32_t* trace, const void* wpart, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA) return cudaErrorNotSupported;   // other modes: own kernels
  const LeafOut none = {};
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? prefill_typed<__nv_bfloat16, 128>(p, Q, K, V, tree, q_start, n_q, O, trace, wpart, none, s)
                      : prefill_typed<__nv_bfloat16, 64>(p, Q, K, V, tree, q_start, n_q, O, trace, wpart, none, s);
  return p.d == 128 ? prefill_typed<float, 128>(p, Q, K, V, tree, q_start, n_q, O, trace, wpart, none, s)
                    : prefill_typed<float, 64>(p, Q, K, V, tree, q_start, n_q, O, trace, wpart, none, s);
}

cudaError_t launch_prefill_warp_leafout(const Params& p, const void* Q, const void* K,
                                        const void* V, const void* tree, int64_t q_start,
                                        int32_t n_q, int32_t* trace, const void* wpart,
                                        const LeafOut& lo, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA || !lo.counts) return cudaErrorNotSupported;
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? prefill_typed<__nv_bfloat16, 128>(p, Q, K, V, tree, q_start, n_q, nullptr, trace, wpart, lo, s)
                      : prefill_typed<__nv_bfloat16, 64>(p, Q, K, V, tree, q_start, n_q, nullptr, trace, wpart, lo, s);
  return p.d == 128 ? prefill_typed<float, 128>(p, Q, K, V, tree, q_start, n_q, nullptr, trace, wpart, lo, s)
                    : prefill_typed<float, 64>(p, Q, K, V, tree, q_start, n_q, nullptr, trace, wpart, lo, s);
}

}  // namespace recsa
