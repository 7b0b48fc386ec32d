// Prefill traversal regrouped by parent node: the tree levels of a prefill
// chunk as tensor-core tiles plus a light per-query-head select pass.
//
// At level l a query head's candidates ("Recursive Sparse Attention:
// Million-Token Length Extrapolation at Logarithmic Cost", abstract: at most k
// kept per level, top-down) are runs of at most b consecutive nodes: the b
// children of each node kept at level l + 1 (slot s of the kept list, indices
// s b .. s b + b - 1), then the orphans, the visible children of the first
// parent that is not visible (node v_{l+1} of level l + 1).  At the top level
// the visible nodes are the orphans of the (invisible) parent 0.  So every run
// is "the children of parent P at level l + 1", and the same run is read by
// every query head that kept P.  With candidate-local RoPE the logit of
// candidate i = i0 + j of a run starting at index i0 is
//   < R(c_l) q, R(i0 + j) key > = < R(c_l - i0) q, R(j) key >:
// the key side is rotated by its offset j in the run alone.  Per level:
//   1. count_kernel/scatter: the (query head, run) pairs of the level are
//      grouped by parent P (a counting sort: per-parent counts, prefix sum,
//      scatter);
//   2. score_tc_kernel: one CTA per parent; the b child keys (rotated by j)
//      meet up to 128 pairs' queries (rotated by c_l - i0) in a
//      [128 x d] x [d x b] tcgen05 product; the operands enter as high and low
//      TF32 parts (3 products), so the scores keep fp32 accuracy and the
//      selection is decided as an fp32 computation would decide it;
//   3. select_kernel: one warp per query head reads its c_l scores, keeps the
//      top k (ties to the lower index), folds the unselected candidates'
//      summaries into its partial softmax (fp32, CUDA cores), and emits the
//      next level's runs (or, at level 1, the kept leaves for the leaf path).
#include "recsa_internal.cuh"
#include "tc05.cuh"

namespace recsa {
namespace {

constexpr int kTThreads = 256;
constexpr int kTTile = 128;                                  // pairs per tile
constexpr int kSelRegSlots = 8;                              // candidates <= 8 x 32
constexpr unsigned long long kTreeWaitNs = 200000000ull;

// Workspace of the tree levels.
struct TreeBufs {
  float* scores;     // [rows][cmax]: the current level's logits
  int* kept;         // [2][rows][kmax]: kept nodes of the last two levels (by parity)
  int4* stage;       // [rows][kmax + 1]: the next level's runs {row, i0 | n << 16, rot, run}
  int2* spos;        // [rows][kmax + 1]: {bucket, position in the bucket}
  int* nruns;        // [rows]
  int4* pairs;       // [rows * (kmax + 1)]: runs grouped by parent
  float* runpart;    // [rows][kmax + 1][d]: per run, sum_j exp(s_j - m_run) value_j
  float2* runml;     // [rows][kmax + 1]: per run, (m_run, sum_j exp(s_j - m_run))
  int* counts;       // per level l: [batch][hkv][np_l] at cbase[l]
  int* offsets;
  int64_t cbase[kMaxLevels + 2];
  int np[kMaxLevels + 2];        // parents per (sequence, KV head) whose children are at level l
  int cmax, kmax;
};

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

int tree_kmax(const Params& p) {
  const int64_t n1 = p.lay.levels > 0 ? p.lay.nodes[0] : 0;
  const int64_t k = p.k < n1 ? p.k : n1;
  return int(k < 1 ? 1 : k);
}

int tree_cmax(const Params& p) {
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t cm = int64_t(p.b) * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  return int(cm < 1 ? 1 : cm);
}

TreeBufs tree_carve(const Params& p, int32_t n_q, void* ws, size_t* total) {
  TreeBufs t = {};
  const size_t rows = size_t(p.batch) * n_q * p.hq;
  t.kmax = tree_kmax(p);
  t.cmax = (tree_cmax(p) + 3) / 4 * 4;
  size_t nb = 0;
  for (int l = 1; l <= p.lay.levels; ++l) {
    t.np[l] = int(p.lay.nodes[l - 1] / p.b + 1);
    t.cbase[l] = int64_t(nb);
    nb += size_t(p.batch) * p.hkv * t.np[l];
  }
  const size_t runs = rows * (t.kmax + 1);
  size_t off[11];
  off[0] = 0;                                           // scores
  off[1] = al256(off[0] + rows * t.cmax * 4);           // kept
  off[2] = al256(off[1] + 2 * rows * t.kmax * 4);       // stage
  off[3] = al256(off[2] + runs * 16);                   // spos
  off[4] = al256(off[3] + runs * 8);                    // nruns
  off[5] = al256(off[4] + rows * 4);                    // pairs
  off[6] = al256(off[5] + runs * 16);                   // counts
  off[7] = al256(off[6] + nb * 4);                      // offsets
  off[8] = al256(off[7] + nb * 4);                      // runpart
  off[9] = al256(off[8] + runs * p.d * 4);              // runml
  off[10] = al256(off[9] + runs * 8);
  if (total) *total = off[10];
  if (ws) {
    char* b = reinterpret_cast<char*>(ws);
    t.scores = reinterpret_cast<float*>(b + off[0]);
    t.kept = reinterpret_cast<int*>(b + off[1]);
    t.stage = reinterpret_cast<int4*>(b + off[2]);
    t.spos = reinterpret_cast<int2*>(b + off[3]);
    t.nruns = reinterpret_cast<int*>(b + off[4]);
    t.pairs = reinterpret_cast<int4*>(b + off[5]);
    t.counts = reinterpret_cast<int*>(b + off[6]);
    t.offsets = reinterpret_cast<int*>(b + off[7]);
    t.runpart = reinterpret_cast<float*>(b + off[8]);
    t.runml = reinterpret_cast<float2*>(b + off[9]);
  }
  return t;
}

__device__ __forceinline__ unsigned order_key_f(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp per query head (row).  L: the level selected here (L > top: no
// selection); emits the runs of level L - 1 (or the kept leaves at L = 1).
template <int D>
__global__ void __launch_bounds__(256, 4)
select_kernel(Params p, TreeBufs tb, LeafOut lo, const void* __restrict__ tree, int L,
              int64_t q_start, int n_q, int32_t* __restrict__ trace) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int row = int(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int rows = p.batch * n_q * p.hq;      // < 2^31 (checked on the host)
  if (row >= rows) return;
  const int h = row % p.hq;
  const int qi = (row / p.hq) % n_q;
  const int seq = row / (p.hq * n_q);
  const int g = h / p.group;
  const int64_t t = q_start + qi;
  // closed-form visibility and counts, top down: c_l = b kappa_{l+1} + (v_l -
  // b v_{l+1}), kappa_l = min(k, c_l), v_l = floor(a / b^(l-1)); only the
  // levels around L are kept (no per-level arrays); positions fit 31 bits
  const int a = int((t + 1 - p.W > 0 ? t + 1 - p.W : 0) / p.B);
  auto vis_at = [&](int per_log, int per) -> int {   // a / b^(lev-1)
    return p.bsh >= 0 ? a >> per_log : a / per;
  };
  int top = 0, pertop = 1, plogtop = 0;
  {
    int per = 1, plog = 0;
    for (int lev = 1; lev <= p.lay.levels; ++lev) {
      if (a < per) break;
      top = lev;
      pertop = per;
      plogtop = plog;
      if (per > a / p.b) break;
      per *= p.b;
      plog += p.bsh;
    }
  }
  int cL = 0, kL = 0, kL1 = 0, cLm = 0;
  int vL1 = 0, vL = 0, vLm = 0;
  {
    int kup = 0, vup = 0, per = pertop, plog = plogtop;
    const int lo_lev = L - 1 > 1 ? L - 1 : 1;
    for (int lev = top; lev >= lo_lev; --lev) {
      const int v = vis_at(plog, per);
      const int c = p.b * kup + (v - p.b * vup);
      const int kk = c < p.k ? c : p.k;
      if (lev == L + 1) {
        kL1 = kk;
        vL1 = v;
      }
      if (lev == L) {
        cL = c;
        kL = kk;
        vL = v;
      }
      if (lev == L - 1) {
        cLm = c;
        vLm = v;
      }
      kup = kk;
      vup = v;
      per /= p.b;
      plog -= p.bsh;
    }
  }
  const int kmax = tb.kmax;
  const int tstride = kTraceHead + kMaxLevels * p.k;
  int* keptL = tb.kept + int64_t(L & 1) * rows * kmax + int64_t(row) * kmax;
  const int* keptUp = tb.kept + int64_t((L + 1) & 1) * rows * kmax + int64_t(row) * kmax;

  if (L <= top) {
    const int c = cL, kap = kL;
    const int kup = L < top ? kL1 : 0;
    const int vup = vL1;
    const float* sc = tb.scores + int64_t(row) * tb.cmax;
    const float* vals = level_vals(p, const_cast<void*>(tree), L, seq, g);
    // candidate i -> node: children of the kept parents, then the orphans
    auto node_of = [&](int i) -> int {
      if (i < p.b * kup) return keptUp[div_b(p, i)] * p.b + mod_b(p, i);
      return p.b * vup + (i - p.b * kup);
    };
    float sv[kSelRegSlots];
    unsigned key[kSelRegSlots];
#pragma unroll
    for (int s = 0; s < kSelRegSlots; ++s) {
      const int i = s * 32 + lane;
      sv[s] = i < c ? sc[i] : -INFINITY;
      key[s] = i < c ? order_key_f(sv[s]) : 0u;
    }
    // top-k: kap rounds of a warp arg-max (ties -> lower index)
    unsigned taken = 0;
    if (kap >= c) {
#pragma unroll
      for (int s = 0; s < kSelRegSlots; ++s)
        if (s * 32 + lane < c) taken |= 1u << s;
    } else {
      for (int r = 0; r < kap; ++r) {
        unsigned bk = key[0];
        int bs = 0;
#pragma unroll
        for (int s = 1; s < kSelRegSlots; ++s)
          if (key[s] > bk) {
            bk = key[s];
            bs = s;
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
          for (int s = 0; s < kSelRegSlots; ++s)
            if (s == bs) key[s] = 0u;
        }
      }
    }
    // kept list in index order
    int cnt = 0;
    const int ns = (c + 31) >> 5;
    for (int s = 0; s < ns; ++s) {
      const int i = s * 32 + lane;
      const bool f = i < c && ((taken >> s) & 1u);
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (f) {
        const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
        const int node = node_of(i);
        keptL[pos] = node;
        if (trace) trace[int64_t(row) * tstride + kTraceHead + (L - 1) * p.k + pos] = node;
      }
      cnt += __popc(bal);
    }
    // fold the unselected candidates' summaries into the partial softmax: the
    // score tiles left, per run r, U_r = sum_j exp(s_j - m_r) value_j over all
    // of its children and L_r = sum_j exp(s_j - m_r); the unselected part is
    // sum_r exp(m_r - M) (U_r, L_r) minus exp(s_i - M) (value_i, 1) for each
    // kept candidate i
    if (kap < c) {
      const int nrun = kup + ((vL - p.b * vL1) > 0 ? 1 : 0);
      const int64_t rb = int64_t(row) * (kmax + 1);
      float2 mr = lane < nrun ? tb.runml[rb + lane] : make_float2(-INFINITY, 0.f);
      float mx = mr.x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float* prow = lo.part + int64_t(row) * (D + 2);
      const float2 ml = *reinterpret_cast<const float2*>(prow + D);
      const float Mn = fmaxf(ml.x, mx);
      float ua[PER], ka[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) ua[e] = ka[e] = 0.f;
      float ul = 0.f, kl = 0.f;
      // all runs
      for (int r = 0; r < nrun; ++r) {
        const float mrr = __shfl_sync(0xffffffffu, mr.x, r);
        const float lrr = __shfl_sync(0xffffffffu, mr.y, r);
        const float w = __expf(mrr - Mn);
        const float* ur = tb.runpart + (rb + r) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 x = *reinterpret_cast<const float4*>(ur);
          ua[0] = fmaf(w, x.x, ua[0]);
          ua[1] = fmaf(w, x.y, ua[1]);
          ua[2] = fmaf(w, x.z, ua[2]);
          ua[3] = fmaf(w, x.w, ua[3]);
        } else {
          const float2 x = *reinterpret_cast<const float2*>(ur);
          ua[0] = fmaf(w, x.x, ua[0]);
          ua[1] = fmaf(w, x.y, ua[1]);
        }
        ul = fmaf(w, lrr, ul);
      }
      // the kept candidates (at most k, their rows loaded together)
#pragma unroll
      for (int s = 0; s < kSelRegSlots; ++s) {
        if (s * 32 >= c) break;
        const int i = s * 32 + lane;
        const bool sel = i < c && ((taken >> s) & 1u);
        const float w = sel ? __expf(sv[s] - Mn) : 0.f;
        const int node = sel ? node_of(i) : 0;
        unsigned m = __ballot_sync(0xffffffffu, sel);
        while (m) {
          constexpr int U = 8;
          float ws[U];
          int nd[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int src = m ? __ffs(m) - 1 : 0;
            const bool real = m != 0;
            m &= m - 1;
            ws[u] = real ? __shfl_sync(0xffffffffu, w, src) : 0.f;
            nd[u] = __shfl_sync(0xffffffffu, node, src);
            if (!real) nd[u] = 0;
          }
          float v[U][PER];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const float* vr = vals + int64_t(nd[u]) * D + lane * PER;
            if constexpr (PER == 4) {
              const float4 x = *reinterpret_cast<const float4*>(vr);
              v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
            } else {
              const float2 x = *reinterpret_cast<const float2*>(vr);
              v[u][0] = x.x; v[u][1] = x.y;
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int e = 0; e < PER; ++e) ka[e] = fmaf(ws[u], v[u][e], ka[e]);
            kl += ws[u];
          }
        }
      }
      // the unselected mass; below fp32 resolution of the runs' mass it is dropped
      float dl = ul - kl;
      const bool keep = dl > 1e-6f * ul;
      const float scale = ml.x == -INFINITY ? 0.f : __expf(ml.x - Mn);
      const float lsum = ml.y * scale + (keep ? dl : 0.f);
      const float il = 1.f / lsum;
#pragma unroll
      for (int e = 0; e < PER; ++e)
        prow[lane * PER + e] =
            (prow[lane * PER + e] * ml.y * scale + (keep ? ua[e] - ka[e] : 0.f)) * il;
      __syncwarp();
      if (lane == 0) *reinterpret_cast<float2*>(prow + D) = make_float2(Mn, lsum);
      __syncwarp();
    }
  }

  // emit the runs of level L - 1
  const int Ln = L - 1;
  if (Ln >= 1 && top >= Ln) {
    const int kprev = L <= top ? kL : 0;
    const int cn = cLm;
    const int orph = vLm - p.b * vL;
    const int nrun = kprev + (orph > 0 ? 1 : 0);
    const int64_t hb = (int64_t(seq) * p.hkv + g) * tb.np[Ln];
    for (int r = lane; r < nrun; r += 32) {
      const int P = r < kprev ? keptL[r] : vL;
      const int i0 = r < kprev ? r * p.b : p.b * kprev;
      const int n = r < kprev ? p.b : orph;
      const int64_t bucket = hb + P;
      const int pos = atomicAdd(tb.counts + tb.cbase[Ln] + bucket, 1);
      tb.stage[int64_t(row) * (kmax + 1) + r] = make_int4(row, i0 | (n << 16), cn - i0, r);
      tb.spos[int64_t(row) * (kmax + 1) + r] = make_int2(int(bucket), pos);
    }
    if (lane == 0) tb.nruns[row] = nrun;
  } else if (Ln >= 1 && lane == 0) {
    tb.nruns[row] = 0;
  }

  // after level 1: the kept leaves for the leaf path, and the trace counts
  if (L == 1) {
    const int nleaf = top >= 1 ? kL : 0;
    const int* kept1 = tb.kept + int64_t(1) * rows * kmax + int64_t(row) * kmax;
    for (int s = lane; s < nleaf; s += 32) {
      const int64_t bucket = (int64_t(seq) * p.hkv + g) * int64_t(lo.nleaf) + kept1[s];
      const int pos = atomicAdd(lo.counts + bucket, 1);
      lo.kept[int64_t(row) * lo.kmax + s] = make_int2(int(bucket), pos);
    }
    if (lane == 0) lo.nkept[row] = nleaf;
    if (trace && lane == 0) {
      const int64_t n_win = t + 1 - int64_t(a) * p.B;
      const int64_t n0 = int64_t(nleaf) * p.B + n_win;
      int32_t* rec = trace + int64_t(row) * tstride;
      for (int lev = top + 1; lev <= kMaxLevels; ++lev) {
        rec[4 + lev - 1] = 0;
        rec[4 + kMaxLevels + lev - 1] = 0;
      }
      int64_t e = 0, rr = 0;
      int kup = 0, vup = 0, per = pertop, plog = plogtop;
      for (int lev = top; lev >= 1; --lev) {
        const int v = vis_at(plog, per);
        const int c = p.b * kup + int(v - p.b * vup);
        const int kk = c < p.k ? c : p.k;
        rec[4 + lev - 1] = c;
        rec[4 + kMaxLevels + lev - 1] = kk;
        e += c - kk;
        rr += c;
        kup = kk;
        vup = v;
        per /= p.b;
        plog -= p.bsh;
      }
      rec[0] = top;
      rec[1] = int32_t(e + n0);
      rec[2] = int32_t(rr + n0);
      rec[3] = int32_t(n0);
    }
  }
}

__global__ void run_scatter_kernel(TreeBufs tb, int64_t rows, int lev) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int kr = tb.kmax + 1;
  if (i >= rows * kr) return;
  const int64_t row = i / kr;
  const int r = int(i % kr);
  if (r >= tb.nruns[row]) return;
  const int2 sp = tb.spos[i];
  tb.pairs[tb.offsets[tb.cbase[lev] + sp.x] + sp.y] = tb.stage[i];
}

// Exclusive prefix sum of n counts (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024) tree_scan_kernel(const int* __restrict__ counts,
                                                         int* __restrict__ offsets, int64_t n) {
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x;
  const int64_t per = (n + 1023) / 1024;
  const int64_t b0 = int64_t(tid) * per;
  const int64_t b1 = b0 + per < n ? b0 + per : n;
  int s = 0;
  for (int64_t i = b0; i < b1; ++i) s += counts[i];
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

__device__ __forceinline__ int kmaj4(int R, int r, int k) { return (k >> 2) * 16 * R + r * 16 + (k & 3) * 4; }

__device__ __forceinline__ void split_store4(unsigned char* dst, int lo_off, float a, float b,
                                             float c, float d) {
  const float ha = tc05::to_tf32(a), hb = tc05::to_tf32(b), hc = tc05::to_tf32(c),
              hd = tc05::to_tf32(d);
  *reinterpret_cast<float4*>(dst) = make_float4(ha, hb, hc, hd);
  *reinterpret_cast<float4*>(dst + lo_off) =
      make_float4(tc05::to_tf32(a - ha), tc05::to_tf32(b - hb), tc05::to_tf32(c - hc),
                  tc05::to_tf32(d - hd));
}

// Rotate 8 rotate-half pairs at frequencies j0.. by table row `idx` and store
// their high and low TF32 parts as row r of a K-major operand of R rows.
__device__ __forceinline__ void rot_split_store(const Params& p, const float2* rope, int idx,
                                                int j0, const float* x1, const float* x2,
                                                unsigned char* base, int lo_off, int R, int r) {
  const int half = p.d / 2;
  float y1[8], y2[8];
  if (p.rope) {
    const float4* cs = reinterpret_cast<const float4*>(rope + int64_t(idx) * half + j0);
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
    split_store4(base + kmaj4(R, r, j0 + 4 * c), lo_off, y1[4 * c], y1[4 * c + 1], y1[4 * c + 2],
                 y1[4 * c + 3]);
    split_store4(base + kmaj4(R, r, half + j0 + 4 * c), lo_off, y2[4 * c], y2[4 * c + 1],
                 y2[4 * c + 2], y2[4 * c + 3]);
  }
}

template <int D, int NB>
struct ScoreSmem {
  static constexpr int kAn = kTTile * D * 4;          // one TF32 part of the queries
  static constexpr int kBn = NB * D * 4;              // one part of the child keys
  static constexpr int kA2n = kTTile * NB * 4;        // one part of the probabilities
  static constexpr int kB2n = D * NB * 4;             // one part of the child values^T
  static constexpr int kA = 0;
  static constexpr int kB = kA + 2 * kAn;
  static constexpr int kA2 = kB + 2 * kBn;
  static constexpr int kB2 = kA2 + 2 * kA2n;
  static constexpr int kDst = kB2 + 2 * kB2n;           // per tile row: run partial offset
  static constexpr int kBar = kDst + kTTile * 8;
  static constexpr int kTotal = kBar + 32;
  static constexpr bool kFits = kTotal <= 227 * 1024;
};

// One CTA per parent P (sequence, KV head, level-(l+1) node) and tile split:
// its children's keys at level l, rotated by their offset j, against tiles of
// 128 pairs' queries rotated by c_l - i0.  The scores go to
// tb.scores[row][i0 + j]; then, per pair, P_j = exp(s_j - m) over its n
// children (m their maximum) meets the children's values in a second product,
// and U = P V and (m, sum P) are written as the run's partial, which the
// select pass folds after removing the kept children.
template <typename T, int D, int NB>
__global__ void __launch_bounds__(kTThreads, 1)
score_tc_kernel(Params p, const T* __restrict__ Q, void* tree, TreeBufs tb, int lev) {
  using S = ScoreSmem<D, NB>;
  constexpr int HALF = D / 2;
  const int64_t b = blockIdx.x;
  const int split = blockIdx.y, nsplit = gridDim.y;   // tiles split, nsplit, ... of the parent
  const int cnt = tb.counts[tb.cbase[lev] + b];
  if (cnt <= split * kTTile) return;
  const int off = tb.offsets[tb.cbase[lev] + b];
  const int np = tb.np[lev];
  const int64_t sg = b / np;                     // seq * hkv + g
  const int P = int(b % np);
  const int64_t seq = sg / p.hkv;
  const int g = int(sg % p.hkv);
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S::kBar);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + S::kBar + 16);
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr uint32_t kCols = 256;                // scores in [0, NB), U in [32, 32 + D)
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
  // the parent's children (rows past the level's nodes are zero): keys rotated
  // by j, values transposed ([d][child])
  const float* keys = level_keys(p, tree, lev, seq, g);
  const float* vals = level_vals(p, tree, lev, seq, g);
  const int64_t nlev = p.lay.nodes[lev - 1];
  for (int task = tid; task < NB * (HALF / 8); task += kTThreads) {
    const int j = task % NB, c = task / NB;
    float x1[8], x2[8];
    const int64_t node = int64_t(P) * p.b + j;
    if (j < p.b && node < nlev) {
      const float* kr = keys + node * D;
      const float4 a0 = *reinterpret_cast<const float4*>(kr + 8 * c);
      const float4 a1 = *reinterpret_cast<const float4*>(kr + 8 * c + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(kr + HALF + 8 * c);
      const float4 b1 = *reinterpret_cast<const float4*>(kr + HALF + 8 * c + 4);
      x1[0] = a0.x; x1[1] = a0.y; x1[2] = a0.z; x1[3] = a0.w;
      x1[4] = a1.x; x1[5] = a1.y; x1[6] = a1.z; x1[7] = a1.w;
      x2[0] = b0.x; x2[1] = b0.y; x2[2] = b0.z; x2[3] = b0.w;
      x2[4] = b1.x; x2[5] = b1.y; x2[6] = b1.z; x2[7] = b1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x1[e] = x2[e] = 0.f;
    }
    rot_split_store(p, rope, j < p.b ? j : 0, 8 * c, x1, x2, sm + S::kB, S::kBn, NB, j);
  }
  for (int task = tid; task < D * (NB / 4); task += kTThreads) {
    const int n = task % D, jq = task / D;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * jq + e;
      const int64_t node = int64_t(P) * p.b + j;
      v[e] = (j < p.b && node < nlev) ? vals[node * D + n] : 0.f;
    }
    split_store4(sm + S::kB2 + kmaj4(D, n, 4 * jq), S::kB2n, v[0], v[1], v[2], v[3]);
  }
  tc05::fence_smem_to_async();
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = *tslot, tU = tmem + 32;
  const uint32_t aA = tc05::smem_u32(sm + S::kA), aB = tc05::smem_u32(sm + S::kB);
  const uint32_t aA2 = tc05::smem_u32(sm + S::kA2), aB2 = tc05::smem_u32(sm + S::kB2);
  constexpr uint32_t id1 = tc05::idesc(tc05::kFmtTF32, kTTile, NB);
  constexpr uint32_t id2 = tc05::idesc(tc05::kFmtTF32, kTTile, D);
  const float inv_sqrt_d = p.inv_sqrt_d;
  bool ok = true;
  unsigned phase = 0;
  for (int t0 = split * kTTile; t0 < cnt && ok; t0 += nsplit * kTTile) {
    const int nt = cnt - t0 < kTTile ? cnt - t0 : kTTile;
    // gather: every load of this thread's tasks is issued before any store
    constexpr int NT = kTTile * (HALF / 8) / kTThreads;
    int4 prs[NT];
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int r = (tid + it * kTThreads) % kTTile;
      prs[it] = r < nt ? tb.pairs[off + t0 + r] : make_int4(0, 0, 0, 0);
    }
    uint4 qa[NT][2];
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int task = tid + it * kTThreads;
      const int r = task % kTTile, c = task / kTTile;
      if (sizeof(T) == 2 && r < nt) {
        const T* q = Q + int64_t(prs[it].x) * D;
        qa[it][0] = *reinterpret_cast<const uint4*>(q + 8 * c);
        qa[it][1] = *reinterpret_cast<const uint4*>(q + HALF + 8 * c);
      } else {
        qa[it][0] = qa[it][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int it = 0; it < NT; ++it) {
      const int task = tid + it * kTThreads;
      const int r = task % kTTile, c = task / kTTile;
      float x1[8], x2[8];
      const int rot = r < nt ? prs[it].z : 0;
      if (r < nt) {
        if constexpr (sizeof(T) == 2) {
          const uint32_t w1[4] = {qa[it][0].x, qa[it][0].y, qa[it][0].z, qa[it][0].w};
          const uint32_t w2[4] = {qa[it][1].x, qa[it][1].y, qa[it][1].z, qa[it][1].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x1[2 * e] = __uint_as_float(w1[e] << 16);
            x1[2 * e + 1] = __uint_as_float(w1[e] & 0xffff0000u);
            x2[2 * e] = __uint_as_float(w2[e] << 16);
            x2[2 * e + 1] = __uint_as_float(w2[e] & 0xffff0000u);
          }
        } else {
          const T* q = Q + int64_t(prs[it].x) * D;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x1[e] = reinterpret_cast<const float*>(q)[8 * c + e];
            x2[e] = reinterpret_cast<const float*>(q)[HALF + 8 * c + e];
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x1[e] = x2[e] = 0.f;
      }
      rot_split_store(p, rope, rot, 8 * c, x1, x2, sm + S::kA, S::kAn, kTTile, r);
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const uint32_t a = aA + kk * 32 * kTTile, bb = aB + kk * 32 * NB;
        const uint64_t ahi = tc05::desc_kmajor(a, 16 * kTTile, 128);
        const uint64_t alo = tc05::desc_kmajor(a + S::kAn, 16 * kTTile, 128);
        const uint64_t bhi = tc05::desc_kmajor(bb, 16 * NB, 128);
        const uint64_t blo = tc05::desc_kmajor(bb + S::kBn, 16 * NB, 128);
        tc05::mma_tf32(tmem, ahi, bhi, id1, kk > 0);
        tc05::mma_tf32(tmem, ahi, blo, id1, 1);
        tc05::mma_tf32(tmem, alo, bhi, id1, 1);
      }
      tc05::mma_commit(&bar[0]);
    }
    ok = __syncthreads_and(tid != 0 || tc05::mbar_wait_bounded(&bar[0], phase, kTreeWaitNs));
    tc05::fence_after_sync();
    // thread i of warps 0-3 owns row i (TMEM lane i); the loads are
    // warp-collective
    const int myrow = tid;
    const bool rowthr = warp < 4;
    float m = -INFINITY, l = 0.f;
    int4 pr = make_int4(0, 0, 0, 0);
    if (ok && warp < 4) {
      float s[NB];
#pragma unroll
      for (int c = 0; c < NB / 16; ++c)
        tc05::tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + 16 * c, s + 16 * c);
      tc05::tmem_wait_ld();
      int n = 0;
      if (rowthr && myrow < nt) {
        pr = tb.pairs[off + t0 + myrow];
        const int i0 = pr.y & 0xffff;
        n = pr.y >> 16;
        float* dst = tb.scores + int64_t(pr.x) * tb.cmax + i0;
#pragma unroll
        for (int j = 0; j < NB; ++j) s[j] *= inv_sqrt_d;
        if ((i0 & 3) == 0) {
#pragma unroll
          for (int j = 0; j < NB; j += 4) {
            if (j + 4 <= n) {
              *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (j + e < n) dst[j + e] = s[j + e];
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < NB; ++j)
            if (j < n) dst[j] = s[j];
        }
#pragma unroll
        for (int j = 0; j < NB; ++j)
          if (j < n) m = fmaxf(m, s[j]);
      }
      // P over the run's n children (zero elsewhere and for rows past the tile)
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        s[j] = j < n ? __expf(s[j] - m) : 0.f;
        l += s[j];
      }
      if (rowthr) {
#pragma unroll
        for (int j = 0; j < NB; j += 4)
          split_store4(sm + S::kA2 + kmaj4(kTTile, myrow, j), S::kA2n, s[j], s[j + 1], s[j + 2],
                       s[j + 3]);
      }
    }
    tc05::fence_smem_to_async();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (tid == 0 && ok) {
#pragma unroll
      for (int kk = 0; kk < NB / 8; ++kk) {
        const uint32_t a = aA2 + kk * 32 * kTTile, bb = aB2 + kk * 32 * D;
        const uint64_t ahi = tc05::desc_kmajor(a, 16 * kTTile, 128);
        const uint64_t alo = tc05::desc_kmajor(a + S::kA2n, 16 * kTTile, 128);
        const uint64_t bhi = tc05::desc_kmajor(bb, 16 * D, 128);
        const uint64_t blo = tc05::desc_kmajor(bb + S::kB2n, 16 * D, 128);
        tc05::mma_tf32(tU, ahi, bhi, id2, kk > 0);
        tc05::mma_tf32(tU, ahi, blo, id2, 1);
        tc05::mma_tf32(tU, alo, bhi, id2, 1);
      }
      tc05::mma_commit(&bar[1]);
    }
    ok = __syncthreads_and(tid != 0 || !ok || tc05::mbar_wait_bounded(&bar[1], phase, kTreeWaitNs)) && ok;
    tc05::fence_after_sync();
    // U rows: staged (16-byte chunks rotated by the row) in the query tile's
    // bytes, then stored whole, coalesced
    constexpr int CPR = D / 4;
    unsigned char* stg = sm + S::kA;
    static_assert(kTTile * D * 4 <= S::kAn, "staging fits the query tile");
    if (ok && warp < 4) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc05::tmem_ld16(tU + (uint32_t(warp * 32) << 16) + 32 * c, o);
        tc05::tmem_ld16(tU + (uint32_t(warp * 32) << 16) + 32 * c + 16, o + 16);
        tc05::tmem_wait_ld();
        if (rowthr) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = 8 * c + e;
            *reinterpret_cast<float4*>(stg + myrow * (D * 4) + ((ch + myrow) % CPR) * 16) =
                make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
          }
        }
      }
      if (rowthr && myrow < nt) {
        const int64_t slot = int64_t(pr.x) * (tb.kmax + 1) + pr.w;
        tb.runml[slot] = make_float2(m, l);
        reinterpret_cast<int64_t*>(sm + S::kDst)[myrow] = slot * D;
      }
    }
    __syncthreads();
    if (ok) {
      // destination rows from shared memory: no global load between the stores
      constexpr int RPW = 32 / CPR;
      const int sub = (threadIdx.x & 31) / CPR, ch = (threadIdx.x & 31) % CPR;
      const int64_t* dsts = reinterpret_cast<const int64_t*>(sm + S::kDst);
      for (int r = warp * RPW + sub; r < nt; r += (kTThreads / 32) * RPW) {
        float* dst = tb.runpart + dsts[r];
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
    tc05::mbar_wait_bounded(&bar[0], phase, kTreeWaitNs);
    tc05::mbar_wait_bounded(&bar[1], phase, kTreeWaitNs);
  }
  __syncthreads();
  if (warp == 0) tc05::tmem_dealloc(tmem, kCols);
}

template <typename T, int D, int NB>
cudaError_t score_launch(const Params& p, const void* Q, void* tree, const TreeBufs& tb, int lev,
                         cudaStream_t s) {
  using S = ScoreSmem<D, NB>;
  static_assert(S::kFits, "score tile does not fit");
  auto kern = score_tc_kernel<T, D, NB>;
  cudaError_t e = ensure_smem(kern, S::kTotal);
  if (e != cudaSuccess) return e;
  const int64_t nb = int64_t(p.batch) * p.hkv * tb.np[lev];
  // the upper levels have few parents, each read by many query heads: their
  // tiles are spread over several CTAs so that every level fills the GPU
  int64_t split = (2048 + nb - 1) / nb;
  split = split < 1 ? 1 : split > 256 ? 256 : split;
  kern<<<dim3(unsigned(nb), unsigned(split)), kTThreads, S::kTotal, s>>>(
      p, reinterpret_cast<const T*>(Q), tree, tb, lev);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t score_dispatch(const Params& p, const void* Q, void* tree, const TreeBufs& tb,
                           int lev, cudaStream_t s) {
  if (p.b <= 16) return score_launch<T, D, 16>(p, Q, tree, tb, lev, s);
  if (p.b <= 32) return score_launch<T, D, 32>(p, Q, tree, tb, lev, s);
  return cudaErrorNotSupported;
}

}  // namespace

bool prefill_tree_supported(const Params& p) {
  if (p.mode != RECSA_MODE_RECSA || p.kfmt != RECSA_KEYS_F32 || p.nref != 1) return false;
  if (p.d != 64 && p.d != 128) return false;
  if (p.lay.levels < 1) return false;
  if (tree_cmax(p) > 32 * kSelRegSlots) return false;
  if (p.b > 32 || p.b * int64_t(tree_kmax(p)) >= 65536) return false;
  return true;
}

size_t prefill_tree_workspace_need(const Params& p, int32_t n_q) {
  size_t total = 0;
  tree_carve(p, n_q, nullptr, &total);
  return total;
}

// The tree levels of a prefill call: fills lo.part (window partial on entry)
// with the unselected summaries, and lo.kept / lo.nkept / lo.counts with the
// kept leaves, as the traversal kernel does.
cudaError_t launch_prefill_tree(const Params& p, const void* Q, const void* tree,
                                int64_t q_start, int32_t n_q, int32_t* trace, const LeafOut& lo,
                                void* ws, cudaStream_t s) {
  if (!prefill_tree_supported(p)) return cudaErrorNotSupported;
  const int64_t rows = int64_t(p.batch) * n_q * p.hq;
  if (rows * (tree_kmax(p) + 1) >= (int64_t(1) << 31) || q_start + n_q >= (int64_t(1) << 31))
    return cudaErrorNotSupported;
  const TreeBufs tb = tree_carve(p, n_q, ws, nullptr);
  // deepest level any query of the range reaches
  int dmax = 0;
  {
    const int64_t t = q_start + n_q - 1;
    const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
    const int64_t a = s0 / p.B;
    int64_t per = 1;
    for (int lev = 1; lev <= p.lay.levels; ++lev) {
      if (a / per == 0) break;
      dmax = lev;
      per *= p.b;
    }
  }
  int64_t ncount = 0;
  for (int l = 1; l <= p.lay.levels; ++l) ncount += int64_t(p.batch) * p.hkv * tb.np[l];
  cudaError_t e = cudaMemsetAsync(tb.counts, 0, size_t(ncount) * 4, s);
  if (e != cudaSuccess) return e;
  void* tr = const_cast<void*>(tree);
  const unsigned sblocks = unsigned((rows + 7) / 8);
  auto select = [&](int L) -> cudaError_t {
    if (p.d == 128)
      select_kernel<128><<<sblocks, 256, 0, s>>>(p, tb, lo, tree, L, q_start, n_q, trace);
    else
      select_kernel<64><<<sblocks, 256, 0, s>>>(p, tb, lo, tree, L, q_start, n_q, trace);
    return cudaGetLastError();
  };
  // the first level's runs (queries whose top level is the deepest), then per level
  if (dmax >= 1) {
    e = select(dmax + 1);
    if (e != cudaSuccess) return e;
  }
  for (int lev = dmax; lev >= 1; --lev) {
    const int64_t nb = int64_t(p.batch) * p.hkv * tb.np[lev];
    tree_scan_kernel<<<1, 1024, 0, s>>>(tb.counts + tb.cbase[lev], tb.offsets + tb.cbase[lev],
                                        nb);
    const int64_t tasks = rows * (tb.kmax + 1);
    run_scatter_kernel<<<unsigned((tasks + 255) / 256), 256, 0, s>>>(tb, rows, lev);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.dtype == RECSA_DTYPE_BF16)
      e = p.d == 128 ? score_dispatch<__nv_bfloat16, 128>(p, Q, tr, tb, lev, s)
                     : score_dispatch<__nv_bfloat16, 64>(p, Q, tr, tb, lev, s);
    else
      e = p.d == 128 ? score_dispatch<float, 128>(p, Q, tr, tb, lev, s)
                     : score_dispatch<float, 64>(p, Q, tr, tb, lev, s);
    if (e != cudaSuccess) return e;
    e = select(lev);
    if (e != cudaSuccess) return e;
  }
  if (dmax == 0) {
    // no query of the range sees the tree: no kept leaves, trace counts only
    e = select(1);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace recsa
