// Decode attention on a thread-block cluster per (sequence, query, KV head).
//
// Same method as the generic kernel ("Recursive Sparse Attention:
// Million-Token Length Extrapolation at Logarithmic Cost", abstract: top-down
// selection of at most k candidates per level, unselected summaries in one
// softmax with the exact tokens, candidate-local RoPE), laid out for B200:
//
//   * The CS CTAs of a cluster split every level's (head, candidate) pairs.
//     Each CTA scores its share and stores the scores into every CTA's shared
//     memory (distributed shared memory); one cluster barrier per level, then
//     each CTA runs the same warp top-k on the full score table, so every CTA
//     knows the kept nodes without a second exchange.
//   * Work that does not depend on the selection (the window tokens) runs in
//     the first pass; the values of a level's unselected candidates are
//     folded in during the next level's pass, so each level costs one
//     dependent memory round trip.
//   * Rows (fp32 summary rows, bf16/fp32 K/V rows) are read straight into
//     registers with 16-byte loads: a row is spread over d/8 lanes, each lane
//     holding four rotate-half pairs (j, j + d/2), so the RoPE rotation is
//     local to the lane.  Each lane slot keeps an online softmax state per
//     head; states are merged across slots, warps and finally the cluster
//     (again through distributed shared memory) without any global scratch.
#include <cooperative_groups.h>

#include "recsa_internal.cuh"
#include "rows.cuh"
#include "pool.cuh"

namespace cg = cooperative_groups;

namespace recsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRegSlots = 8;      // top-k candidates held in registers: 32 per slot
constexpr int kUnroll = 3;
constexpr int kTokUnroll = 3;

enum ItemKind { kKey = 0, kVal = 1, kNone = 2 };

// Fused decode step (append + decode in one launch): the new token, the pooler
// and the per-sequence step counters in the tree header.
struct StepArgs {
  const void* k_new;
  const void* v_new;
  const float* r;
  int64_t r_stride;
  int64_t* len_w;
  int* counters;
  int fuse;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_cluster_kernel(Params p, const T* __restrict__ Q, const T* __restrict__ K,
                      const T* __restrict__ V, const void* __restrict__ tree,
                      const int64_t* __restrict__ len_dev, int n_q, T* __restrict__ O,
                      int32_t* __restrict__ trace, int cmax, int kmax, int wrows,
                      StepArgs st) {
  constexpr int HALF = D / 2, LPR = HALF / 4, SPW = 32 / LPR, NSLOT = kWarps * SPW;
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = int(cluster.num_blocks());
  const int rank = int(cluster.block_rank());
  const int qi = blockIdx.y;
  const int64_t seq = blockIdx.z / p.hkv;
  const int g = int(blockIdx.z % p.hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR;
  const int j0 = 4 * sub;

  extern __shared__ __align__(16) unsigned char smem[];
  float* qf = reinterpret_cast<float*>(smem);          // [G][D] raw query
  float* qlev = qf + G * D;                            // [G][D] rotated to the level's c
  float* qtok = qlev + G * D;                          // [G][D] rotated to n0 - 1
  float* sc = qtok + G * D;                            // [2][G][cmax] scores
  float* wsc = sc + 2 * G * cmax;                      // [kWarps][D + 2] warp merge
  float* wwin = wsc + kWarps * (D + 2);                // [kWarps][G][D + 2] window partials
  float* mrg = wwin + kWarps * G * (D + 2);            // [CS][G][D + 2] cluster merge (rank 0)
  int* kept = reinterpret_cast<int*>(mrg + CS * G * (D + 2));   // [2][G][kmax]
  unsigned char* kfl = reinterpret_cast<unsigned char*>(kept + 2 * G * kmax);  // [2][G][cmax]
  // window rows of this CTA staged by cp.async: K then V, [wrows][D] each
  T* winK = reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(kfl + 2 * G * cmax) + 15) &
                                 ~uintptr_t(15));
  T* winV = winK + size_t(wrows) * D;

  // Fused step: the new token is appended at len (this kernel writes it and
  // pools what it completes), and the query sits on it.  A full sequence is
  // flagged and decoded without the append, as recsa_append would leave it.
  const int64_t len0 = len_dev[seq];
  const bool do_append = st.fuse && len0 >= 0 && len0 < p.cap;
  const int64_t t = do_append ? len0 : len0 - 1;
  const T* knew = reinterpret_cast<const T*>(st.k_new) + (seq * p.hkv + g) * D;
  const T* vnew = reinterpret_cast<const T*>(st.v_new) + (seq * p.hkv + g) * D;
  const int64_t qrow = ((seq * n_q + qi) * p.hq + int64_t(g) * G) * D;
  const bool empty = t < 0 || t >= p.cap;   // uniform over the cluster
  const float2* rope = rope_table(p, tree);
  const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
  const int64_t a = empty ? 0 : s0 / p.B;
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
  // Candidate and kept counts per level: the same for every head.
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
  const int64_t n_win = empty ? 0 : t + 1 - a * p.B;
  const int64_t n0 = int64_t(nleaf) * p.B + n_win;

  for (int x = tid; x < G * D; x += kThreads)
    qf[x] = empty ? 0.f : load_elem(Q, qrow + x, p.dtype);
  __syncthreads();
  auto rotate_q = [&](float* dst, int64_t idx) {
    for (int x = tid; x < G * HALF; x += kThreads) {
      const int h = x / HALF, j = x % HALF;
      const float x1 = qf[h * D + j], x2 = qf[h * D + j + HALF];
      if (p.rope) {
        const float2 cs = rope[idx * HALF + j];
        dst[h * D + j] = x1 * cs.x - x2 * cs.y;
        dst[h * D + j + HALF] = x2 * cs.x + x1 * cs.y;
      } else {
        dst[h * D + j] = x1;
        dst[h * D + j + HALF] = x2;
      }
    }
  };
  if (!empty) rotate_q(qtok, n0 - 1 > 0 ? n0 - 1 : 0);

  // Warps are specialised by head: warps [h * WPH, (h + 1) * WPH) serve query
  // head h of the group, so every lane slot keeps one online-softmax state.
  constexpr int WPH = kWarps / G, HSLOT = WPH * SPW;
  const int hw = warp / WPH;                          // this warp's head
  const int hs = (warp % WPH) * SPW + lane / LPR;     // slot index within the head's warps
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  auto fold = [&](float s, const float* v) {
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
  };

  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  const float inv_sqrt_d = p.inv_sqrt_d;
  const int tstride = kTraceHead + kMaxLevels * p.k;

  // Node id of candidate i of head h at level lev (kept list of lev + 1 in kept[par]).
  auto cand_node = [&](int lev, int h, int i) -> int {
    const int kup = lev < top ? cnt_k[lev + 1] : 0;
    const int vup = lev < top ? int(vis[lev + 1]) : 0;
    if (i < p.b * kup)
      return kept[((lev + 1) & 1) * G * kmax + h * kmax + div_b(p, i)] * p.b + mod_b(p, i);
    return p.b * vup + (i - p.b * kup);
  };
  auto share = [&](int tot, int& lo, int& hi) {
    const int ch = (tot + CS - 1) / CS;
    lo = min(tot, rank * ch);
    hi = min(tot, lo + ch);
  };

  // Window rows [w_lo, w_hi): every slot of the CTA takes rows, each row is
  // loaded, rotated and scored once for all G heads.  The per-slot state of
  // all heads is merged across the warp and left in wwin[warp][G].
  auto window_loop = [&](int w_lo, int w_hi) {
    float mW[G], lW[G], accW[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mW[h] = -INFINITY;
      lW[h] = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) accW[h][c] = 0.f;
    }
    const int nw = w_hi - w_lo;
    const int widx0 = nleaf * p.B + w_lo;
    const int gslot = warp * SPW + lane / LPR;
    // Rows come from the staged copy in shared memory; the slot's RoPE index
    // grows by NSLOT per row, so its (cos, sin) advance by a fixed rotation.
    float csc[8], cstep[8];
    const int rmax = p.lay.rope_rows - 1;
    const bool recur = NSLOT <= rmax;   // the step rotation is a table row
    if (p.rope && recur) {
      load_cs(rope, min(widx0 + gslot, rmax), HALF, j0, csc);
      load_cs(rope, NSLOT, HALF, j0, cstep);
    }
    for (int base = 0; base < nw; base += NSLOT) {
      {
        const int e = base + gslot;
        const bool on = e < nw;
        float xk[8], xv[8];
        const int ee = on ? e : 0;
        SharedPairs<T, HALF>::load(winK + size_t(ee) * D, j0, xk);
        SharedPairs<T, HALF>::load(winV + size_t(ee) * D, j0, xv);
        if (p.rope) {
          if (!recur) load_cs(rope, min(widx0 + e, rmax), HALF, j0, csc);
          rotate8(xk, csc);
          if (recur) advance_cs(csc, cstep);
        }
        const bool on_u = on;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* qv = qtok + h * D;
          float s = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            s = fmaf(qv[j0 + c], xk[c], s);
            s = fmaf(qv[HALF + j0 + c], xk[4 + c], s);
          }
          s = slot_sum<LPR>(s) * inv_sqrt_d;
          if (on_u) {
            if (s > mW[h]) {
              const float r = __expf(mW[h] - s);
              lW[h] = lW[h] * r + 1.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) accW[h][c] = fmaf(accW[h][c], r, xv[c]);
              mW[h] = s;
            } else {
              const float w = __expf(s - mW[h]);
              lW[h] += w;
#pragma unroll
              for (int c = 0; c < 8; ++c) accW[h][c] = fmaf(w, xv[c], accW[h][c]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, mW[h], o);
        const float lo = __shfl_xor_sync(0xffffffffu, lW[h], o);
        const float mn = fmaxf(mW[h], mo);
        const float ra_ = (mW[h] == -INFINITY) ? 0.f : __expf(mW[h] - mn);
        const float rb_ = (mo == -INFINITY) ? 0.f : __expf(mo - mn);
        lW[h] = lW[h] * ra_ + lo * rb_;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float ao = __shfl_xor_sync(0xffffffffu, accW[h][c], o);
          accW[h][c] = accW[h][c] * ra_ + ao * rb_;
        }
        mW[h] = mn;
      }
      if (lane < LPR) {
        float* w = wwin + (warp * G + h) * (D + 2);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          w[j0 + c] = accW[h][c];
          w[HALF + j0 + c] = accW[h][4 + c];
        }
        if (lane == 0) {
          w[D] = mW[h];
          w[D + 1] = lW[h];
        }
      }
    }
  };

  // Tree rows of head hw (this CTA's share): the key candidates of level klev
  // (scored, scores broadcast to every CTA) and the unselected candidates of
  // level vlev (values folded into the softmax).
  auto tree_loop = [&](int klev, int vlev) {
    int k_lo = 0, k_hi = 0, v_lo = 0, v_hi = 0;
    if (klev > 0) share(cnt_c[klev], k_lo, k_hi);
    if (vlev > 0) share(cnt_c[vlev], v_lo, v_hi);
    const int nk = k_hi - k_lo, nv = v_hi - v_lo, total = nk + nv;
    const float* keys = klev > 0 ? level_keys(p, const_cast<void*>(tree), klev, seq, g) : nullptr;
    const float* vals = vlev > 0 ? level_vals(p, const_cast<void*>(tree), vlev, seq, g) : nullptr;
    const int kupK = (klev > 0 && klev < top) ? cnt_k[klev + 1] : 0;
    const int nchK = p.b * kupK;
    const int orphK = (klev > 0 && klev < top) ? p.b * int(vis[klev + 1]) - nchK : 0;
    const int* keptK = kept + ((klev + 1) & 1) * G * kmax + hw * kmax;
    const int kupV = (vlev > 0 && vlev < top) ? cnt_k[vlev + 1] : 0;
    const int nchV = p.b * kupV;
    const int orphV = (vlev > 0 && vlev < top) ? p.b * int(vis[vlev + 1]) - nchV : 0;
    const int* keptV = kept + ((vlev + 1) & 1) * G * kmax + hw * kmax;
    const float* scV = sc + (vlev & 1) * G * cmax + hw * cmax;
    const unsigned char* flV = kfl + (vlev & 1) * G * cmax + hw * cmax;
    float* scK = sc + (klev & 1) * G * cmax + hw * cmax;
    const float* ql = qlev + hw * D;
    // key items step their RoPE index by HSLOT per slot: seeded once per batch
    const int rmax = p.lay.rope_rows - 1;
    float cstep[8];
    if (p.rope) load_cs(rope, HSLOT, HALF, j0, cstep);
    for (int base = 0; base < total; base += HSLOT * kUnroll) {
      RawPairs ra[kUnroll];
      float csc[8];
      int kind[kUnroll], idx[kUnroll];
      if (p.rope) load_cs(rope, min(k_lo + base + hs, rmax), HALF, j0, csc);
      float sv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = base + u * HSLOT + hs;
        kind[u] = kNone;
        idx[u] = 0;
        sv[u] = 0.f;
        if (e < nk) {
          const int i = k_lo + e;
          const int node = i < nchK ? keptK[div_b(p, i)] * p.b + mod_b(p, i) : orphK + i;
          kind[u] = kKey;
          idx[u] = i;
          RawLoad<float, HALF>::load(keys + int64_t(node) * D, j0, ra[u]);
        } else if (e < total) {
          const int i = v_lo + (e - nk);
          if (!flV[i]) {
            const int node = i < nchV ? keptV[div_b(p, i)] * p.b + mod_b(p, i) : orphV + i;
            kind[u] = kVal;
            sv[u] = scV[i];
            RawLoad<float, HALF>::load(vals + int64_t(node) * D, j0, ra[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        float x[8], s = 0.f;
        RawLoad<float, HALF>::cvt(ra[u], x);
        if (kind[u] == kKey && p.rope) rotate8(x, csc);
        if (p.rope) advance_cs(csc, cstep);
        if (kind[u] == kKey) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            s = fmaf(ql[j0 + c], x[c], s);
            s = fmaf(ql[HALF + j0 + c], x[4 + c], s);
          }
        }
        if (__any_sync(0xffffffffu, kind[u] == kKey)) s = slot_sum<LPR>(s) * inv_sqrt_d;
        if (kind[u] == kKey) {
          float* dstp = scK + idx[u];
          if (sub < CS) *cluster.map_shared_rank(dstp, sub) = s;
          if (sub + LPR < CS) *cluster.map_shared_rank(dstp, sub + LPR) = s;
        } else if (kind[u] == kVal) {
          fold(sv[u], x);
        }
      }
    }
  };

  // Kept-leaf tokens of head hw (this CTA's share), after level 1's top-k.
  auto token_loop = [&]() {
    int t_lo = 0, t_hi = 0;
    share(nleaf * p.B, t_lo, t_hi);
    const int nt = t_hi - t_lo;
    const int* kept1 = kept + 1 * G * kmax + hw * kmax;           // level 1 = parity 1
    const float* qt = qtok + hw * D;
    const int rmax = p.lay.rope_rows - 1;
    float cstep[8];
    if (p.rope) load_cs(rope, HSLOT, HALF, j0, cstep);
    for (int base = 0; base < nt; base += HSLOT * kTokUnroll) {
      TokRow<T, HALF> rk[kTokUnroll], rv[kTokUnroll];
      float csc[8];
      bool on[kTokUnroll];
      if (p.rope) load_cs(rope, min(t_lo + base + hs, rmax), HALF, j0, csc);
#pragma unroll
      for (int u = 0; u < kTokUnroll; ++u) {
        const int e = base + u * HSLOT + hs;
        on[u] = e < nt;
        if (on[u]) {
          const int r = t_lo + e;
          const int pos = kept1[div_B(p, r)] * p.B + mod_B(p, r);
          rk[u].load(K + (kvbase + pos) * D, j0);
          rv[u].load(V + (kvbase + pos) * D, j0);
        }
      }
#pragma unroll
      for (int u = 0; u < kTokUnroll; ++u) {
        float xk[8], xv[8], s = 0.f;
        rk[u].cvt(xk);
        rv[u].cvt(xv);
        if (p.rope) {
          rotate8(xk, csc);
          advance_cs(csc, cstep);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          s = fmaf(qt[j0 + c], xk[c], s);
          s = fmaf(qt[HALF + j0 + c], xk[4 + c], s);
        }
        s = slot_sum<LPR>(s) * inv_sqrt_d;
        if (on[u]) fold(s, xv);
      }
    }
  };

  auto run_pass = [&](int w_lo, int w_hi, int klev, int vlev, bool tokens) {
    if (w_hi > w_lo) {
      cp_async_wait_all();
      __syncthreads();
      window_loop(w_lo, w_hi);
    }
    if (klev > 0 || vlev > 0) tree_loop(klev, vlev);
    if (tokens) token_loop();
  };

  // Top-k of head h at level lev over the full score table (every CTA runs
  // the same selection on the same broadcast scores).  One warp per head
  // takes kap rounds of a warp arg-max: lane l holds the order-preserving
  // keys of candidates l, l + 32, ... in registers (0 = none or taken; every
  // finite score maps above 0); redux.sync gives the round's maximum, a
  // ballot the lanes holding it, and on a tie of keys across lanes the lowest
  // index wins (within a lane the lowest slot).  Bit s of `taken` marks
  // candidate 32 s + l as kept.  Candidates beyond 32 * kRegSlots are read
  // from shared memory in the same rounds.  The kept list is compacted in
  // index order with one ballot per slot row.  The selecting warp of head h
  // is h * WPH + (h % 4), so the G selections run on different schedulers.
  auto topk = [&](int lev) {
    const int c = cnt_c[lev], kap = cnt_k[lev];
    const int par = lev & 1;
    if (warp == hw * WPH + (hw & 3) % WPH) {
      const int h = hw;
      const float* row = sc + par * G * cmax + h * cmax;
      const int ns = (c + 31) >> 5;
      unsigned taken = 0;
      if (kap >= c) {
        for (int s = 0; s < ns; ++s)
          if (s * 32 + lane < c) taken |= 1u << s;
      } else {
        unsigned key[kRegSlots];
#pragma unroll
        for (int s = 0; s < kRegSlots; ++s) {
          const int i = s * 32 + lane;
          key[s] = i < c ? order_key(row[i]) : 0u;
        }
        for (int r = 0; r < kap; ++r) {
          unsigned bk = key[0];
          int bs = 0;
#pragma unroll
          for (int s = 1; s < kRegSlots; ++s)
            if (key[s] > bk) {
              bk = key[s];
              bs = s;
            }
          for (int s = kRegSlots; s < ns; ++s) {
            const int i = s * 32 + lane;
            if (i < c && !((taken >> s) & 1u)) {
              const unsigned kk = order_key(row[i]);
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
            for (int s = 0; s < kRegSlots; ++s)
              if (s == bs) key[s] = 0u;
          }
        }
      }
      unsigned char* fl = kfl + par * G * cmax + h * cmax;
      int* kp = kept + par * G * kmax + h * kmax;
      int cnt = 0;
      for (int s = 0; s < ns; ++s) {
        const int i = s * 32 + lane;
        const bool f = i < c && ((taken >> s) & 1u);
        if (i < c) fl[i] = f;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (f) {
          const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
          const int node = cand_node(lev, h, i);
          kp[pos] = node;
          if (trace && rank == 0) {
            const int64_t rec = ((seq * n_q + qi) * p.hq + int64_t(g) * G + h) * tstride;
            trace[rec + kTraceHead + (lev - 1) * p.k + pos] = node;
          }
          // The next pass reads this node's children (keys and values one
          // level down) or, at level 1, its tokens: start pulling them into
          // L2 now, one bulk prefetch per contiguous run, spread over the
          // cluster's CTAs.
          if ((h * kmax + pos) % CS == rank) {
            if (lev > 1) {
              const unsigned bytes = unsigned(p.b) * D * 4;
              prefetch_l2(level_keys(p, const_cast<void*>(tree), lev - 1, seq, g) +
                              int64_t(node) * p.b * D, bytes);
              prefetch_l2(level_vals(p, const_cast<void*>(tree), lev - 1, seq, g) +
                              int64_t(node) * p.b * D, bytes);
            } else {
              const unsigned bytes = unsigned(p.B) * D * unsigned(sizeof(T));
              prefetch_l2(K + (kvbase + int64_t(node) * p.B) * D, bytes);
              prefetch_l2(V + (kvbase + int64_t(node) * p.B) * D, bytes);
            }
          }
        }
        cnt += __popc(bal);
      }
      // orphans one level down (shared by every head)
      if (lev > 1 && h == 0 && lane == 0 && rank == (CS - 1)) {
        const int64_t o0 = int64_t(p.b) * vis[lev], o1 = vis[lev - 1];
        if (o1 > o0) {
          const unsigned bytes = unsigned(o1 - o0) * D * 4;
          prefetch_l2(level_keys(p, const_cast<void*>(tree), lev - 1, seq, g) + o0 * D, bytes);
          prefetch_l2(level_vals(p, const_cast<void*>(tree), lev - 1, seq, g) + o0 * D, bytes);
        }
      }
    }
    __syncthreads();
  };

  // Window share of this CTA (independent of the selection).
  int w_lo = 0, w_hi = 0;
  {
    const int nw = int(n_win), ch = (nw + CS - 1) / CS;
    w_lo = min(nw, rank * ch);
    w_hi = min(nw, w_lo + ch);
  }
  const bool has_win = w_hi > w_lo;
  // the top level's candidates (keys and values), pulled into L2 by rank 0
  if (top > 0 && rank == 0 && tid == 0) {
    const unsigned bytes = unsigned(vis[top]) * D * 4;
    prefetch_l2(level_keys(p, const_cast<void*>(tree), top, seq, g), bytes);
    prefetch_l2(level_vals(p, const_cast<void*>(tree), top, seq, g), bytes);
  }
  // Stage this CTA's window rows now: they do not depend on the selection,
  // so the copies are in flight during the first level pass.
  {
    constexpr int CPR = D * int(sizeof(T)) / 16;       // 16-byte pieces per row
    const int rows = w_hi - w_lo;
    const int64_t row0 = kvbase + int64_t(a) * p.B + w_lo;
    const int64_t tnew = do_append ? t - (int64_t(a) * p.B + w_lo) : -1;   // new token's row
    for (int x = tid; x < rows * CPR; x += kThreads) {
      const int r = x / CPR, c = x % CPR;
      const T* ks = r == tnew ? knew : K + (row0 + r) * D;
      const T* vs = r == tnew ? vnew : V + (row0 + r) * D;
      cp_async16(reinterpret_cast<char*>(winK + size_t(r) * D) + c * 16,
                 reinterpret_cast<const char*>(ks) + c * 16);
      cp_async16(reinterpret_cast<char*>(winV + size_t(r) * D) + c * 16,
                 reinterpret_cast<const char*>(vs) + c * 16);
    }
    cp_async_commit();
  }
  if (top > 0) {
    rotate_q(qlev, cnt_c[top]);
    __syncthreads();
    run_pass(w_lo, w_hi, top, 0, false);
    cluster.sync();
    topk(top);
    for (int lev = top - 1; lev >= 1; --lev) {
      rotate_q(qlev, cnt_c[lev]);
      __syncthreads();
      run_pass(0, 0, lev, lev + 1, false);
      cluster.sync();
      topk(lev);
    }
    run_pass(0, 0, 0, 1, true);
  } else {
    run_pass(w_lo, w_hi, 0, 0, false);
  }

  // Merge: slots of a warp, then the warps of each head, then the cluster
  // (into rank 0).
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
  if (lane < LPR) {
    float* w = wsc + warp * (D + 2);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      w[j0 + c] = acc[c];
      w[HALF + j0 + c] = acc[4 + c];
    }
    if (lane == 0) {
      w[D] = m;
      w[D + 1] = l;
    }
  }
  __syncthreads();
  // CTA state of each head -> rank 0's merge slot [rank]
  float* dst = cluster.map_shared_rank(mrg, 0) + rank * G * (D + 2);
  for (int x = tid; x < G * D; x += kThreads) {
    const int h = x / D, c = x % D;
    float mm = -INFINITY;
    for (int w = h * WPH; w < (h + 1) * WPH; ++w) mm = fmaxf(mm, wsc[w * (D + 2) + D]);
    if (has_win)
      for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, wwin[(w * G + h) * (D + 2) + D]);
    float aa = 0.f, ll = 0.f;
    for (int w = h * WPH; w < (h + 1) * WPH; ++w) {
      const float* ws = wsc + w * (D + 2);
      const float r = (ws[D] == -INFINITY) ? 0.f : __expf(ws[D] - mm);
      aa = fmaf(ws[c], r, aa);
      ll = fmaf(ws[D + 1], r, ll);
    }
    if (has_win)
      for (int w = 0; w < kWarps; ++w) {
        const float* ws = wwin + (w * G + h) * (D + 2);
        const float r = (ws[D] == -INFINITY) ? 0.f : __expf(ws[D] - mm);
        aa = fmaf(ws[c], r, aa);
        ll = fmaf(ws[D + 1], r, ll);
      }
    dst[h * (D + 2) + c] = aa;
    if (c == 0) {
      dst[h * (D + 2) + D] = mm;
      dst[h * (D + 2) + D + 1] = ll;
    }
  }
  cluster.sync();
  if (rank == 0) {
    for (int x = tid; x < G * D; x += kThreads) {
      const int h = x / D, c = x % D;
      float mm = -INFINITY;
      for (int r = 0; r < CS; ++r) mm = fmaxf(mm, mrg[(r * G + h) * (D + 2) + D]);
      float aa = 0.f, ll = 0.f;
      for (int r = 0; r < CS; ++r) {
        const float* ms = mrg + (r * G + h) * (D + 2);
        const float w = (ms[D] == -INFINITY) ? 0.f : __expf(ms[D] - mm);
        aa = fmaf(ms[c], w, aa);
        ll = fmaf(ms[D + 1], w, ll);
      }
      const float o = (empty || ll == 0.f) ? 0.f : aa / ll;
      store_elem(O, qrow + x, o, p.dtype);
    }
    if (trace && !empty) {
      for (int x = tid; x < G * (kTraceHead + kMaxLevels * p.k); x += kThreads) {
        const int h = x / tstride, f = x % tstride;
        const int64_t rec = ((seq * n_q + qi) * p.hq + int64_t(g) * G + h) * tstride;
        int v = 0;
        if (f == 0) v = top;
        else if (f == 1 || f == 2 || f == 3) {
          int64_t e = 0, r = 0;
          for (int lev = 1; lev <= top; ++lev) { e += cnt_c[lev] - cnt_k[lev]; r += cnt_c[lev]; }
          v = int(f == 1 ? e + n0 : f == 2 ? r + n0 : n0);
        } else if (f < 4 + kMaxLevels) {
          const int lev = f - 4 + 1;
          v = lev <= top ? cnt_c[lev] : 0;
        } else if (f < kTraceHead) {
          const int lev = f - 4 - kMaxLevels + 1;
          v = lev <= top ? cnt_k[lev] : 0;
        } else {
          continue;   // kept ids are written per level below
        }
        trace[rec + f] = v;
      }
    }
  }

  if (st.fuse) {
    // Append: the first query's cluster of each (sequence, KV head) writes the
    // token and pools the leaf and ancestors it completes (none of them is
    // visible to this step's query: they end inside its window).
    if (rank == 0 && qi == 0 && do_append) {
      T* Kw = const_cast<T*>(K) + (kvbase + t) * D;
      T* Vw = const_cast<T*>(V) + (kvbase + t) * D;
      for (int x = tid; x < D; x += kThreads) {
        Kw[x] = knew[x];
        Vw[x] = vnew[x];
      }
      __syncthreads();
      if ((t + 1) % p.B == 0 && warp == 0) {
        constexpr int N = D / 32;
        float rl[N], key[N], val[N];
        load_r<N>(st.r + g * st.r_stride, lane, rl);
        int64_t j = (t + 1) / p.B - 1;
        const int64_t row0 = (kvbase + j * p.B) * D;
        pool_rows<T, N>(K + row0, V + row0, p.B, D, rl, inv_sqrt_d, lane, key, val);
        RowIO<float, N>::store(level_keys(p, const_cast<void*>(tree), 1, seq, g) + j * D, lane,
                               key);
        RowIO<float, N>::store(level_vals(p, const_cast<void*>(tree), 1, seq, g) + j * D, lane,
                               val);
        for (int lev = 2; lev <= p.lay.levels && (j + 1) % p.b == 0; ++lev) {
          j = (j + 1) / p.b - 1;
          __syncwarp();
          const float* ck = level_keys(p, const_cast<void*>(tree), lev - 1, seq, g) + j * p.b * D;
          const float* cv = level_vals(p, const_cast<void*>(tree), lev - 1, seq, g) + j * p.b * D;
          pool_rows<float, N>(ck, cv, p.b, D, rl, inv_sqrt_d, lane, key, val);
          RowIO<float, N>::store(level_keys(p, const_cast<void*>(tree), lev, seq, g) + j * D,
                                 lane, key);
          RowIO<float, N>::store(level_vals(p, const_cast<void*>(tree), lev, seq, g) + j * D,
                                 lane, val);
        }
      }
    }
    // Length: every cluster of the sequence read len at its start; the last
    // one to finish (per-sequence counter) publishes len + 1 and resets it.
    if (rank == 0 && tid == 0) {
      if (!do_append) {
        if (len0 >= p.cap) atomicOr(tree_error_word(const_cast<void*>(tree)),
                                    RECSA_DEVERR_APPEND_FULL);
      } else {
        __threadfence();
        const int done = atomicAdd(st.counters + seq, 1);
        if (done == p.hkv * n_q - 1) {
          st.counters[seq] = 0;
          st.len_w[seq] = len0 + 1;
        }
      }
    }
  }
}

}  // namespace
}  // namespace recsa

namespace recsa {
namespace {

template <typename T, int D, int G>
cudaError_t cluster_typed(const Params& p, const void* Q, const void* K, const void* V,
                          const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                          int32_t* trace, cudaStream_t s, int cs, StepArgs st) {
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  int64_t cm = p.b * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  const int cmax = int(cm < 1 ? 1 : cm);
  const int kmax = int(kk < cmax ? kk : cmax);
  if (cmax > 1024) return cudaErrorNotSupported;
  // window rows staged per CTA: at most ceil((W + B - 1) / cs)
  const int wrows = int((int64_t(p.W) + p.B - 1 + cs - 1) / cs);
  const size_t bytes = (size_t(3) * G * D + size_t(2) * G * cmax + size_t(kWarps) * (D + 2) +
                        size_t(kWarps) * G * (D + 2) +
                        size_t(cs) * G * (D + 2)) * 4 + size_t(2) * G * kmax * 4 +
                       size_t(2) * G * cmax + 16 + size_t(2) * wrows * D * sizeof(T);
  if (bytes > 200 * 1024) return cudaErrorNotSupported;
  auto kern = decode_cluster_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(bytes));
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (int64_t(p.batch) * p.hkv > 65535 || n_q > 65535) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, n_q, unsigned(p.batch * p.hkv));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, reinterpret_cast<const T*>(Q),
                            reinterpret_cast<const T*>(K), reinterpret_cast<const T*>(V), tree,
                            len_dev, int(n_q), reinterpret_cast<T*>(O), trace, cmax, kmax,
                            wrows, st);
}

template <typename T, int D>
cudaError_t cluster_g(const Params& p, const void* Q, const void* K, const void* V,
                      const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                      int32_t* trace, cudaStream_t s, int cs, StepArgs st) {
  switch (p.group) {
    case 1: return cluster_typed<T, D, 1>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st);
    case 2: return cluster_typed<T, D, 2>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st);
    case 4: return cluster_typed<T, D, 4>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t cluster_dispatch(const Params& p, const void* Q, const void* K, const void* V,
                             const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                             int32_t* trace, cudaStream_t s, int cs, StepArgs st) {
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? cluster_g<__nv_bfloat16, 128>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st)
                      : cluster_g<__nv_bfloat16, 64>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st);
  return p.d == 128 ? cluster_g<float, 128>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st)
                    : cluster_g<float, 64>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, cs, st);
}

}  // namespace

int decode_cluster_size(const Params& p, int32_t n_q) {
  const char* env = getenv("RECSA_DECODE_CLUSTER");
  if (env) {
    const int v = atoi(env);
    if (v == 1 || v == 2 || v == 4 || v == 8 || v == 16) return v;
  }
  const int64_t clusters = int64_t(p.batch) * p.hkv * n_q;
  int cs = 2;
  while (cs < 16 && clusters * cs * 2 <= 148) cs *= 2;
  return cs;
}

cudaError_t launch_decode_cluster(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                                  int32_t* trace, cudaStream_t s) {
  StepArgs st = {};
  return cluster_dispatch(p, Q, K, V, tree, len_dev, n_q, O, trace, s,
                          decode_cluster_size(p, n_q), st);
}

cudaError_t launch_decode_step(const Params& p, const void* Q, void* K, void* V,
                               const void* k_new, const void* v_new, int64_t* len_dev,
                               const float* r, int64_t r_stride, void* tree, int32_t n_q,
                               void* O, int32_t* trace, cudaStream_t s) {
  if (p.batch > kStepCounters) return cudaErrorNotSupported;
  StepArgs st;
  st.k_new = k_new;
  st.v_new = v_new;
  st.r = r;
  st.r_stride = r_stride;
  st.len_w = len_dev;
  st.counters = reinterpret_cast<int*>(reinterpret_cast<char*>(tree) + kStepCounterOffset);
  st.fuse = 1;
  return cluster_dispatch(p, Q, K, V, tree, len_dev, n_q, O, trace, s,
                          decode_cluster_size(p, n_q), st);
}

}  // namespace recsa
