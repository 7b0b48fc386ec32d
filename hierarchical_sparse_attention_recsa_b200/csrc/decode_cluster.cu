// Decode attention on a thread-block cluster per (sequence, query, KV head).
//
// Same method as the generic kernel ("Recursive Sparse Attention:
// Million-Token Length Extrapolation at Logarithmic Cost", abstract: top-down
// selection of at most k candidates per level, unselected summaries in one
// softmax with the exact tokens, candidate-local RoPE), laid out for B200:
//
//   * Every gather of the method is a few contiguous runs: a level's
//     candidates are the b children of each kept node (b * d contiguous fp32
//     summary rows) plus one run of orphans, and a kept leaf is B contiguous
//     K rows and B contiguous V rows.  Each run is copied into shared memory
//     by one TMA bulk copy (cp.async.bulk) completing on an mbarrier, so a
//     level's whole candidate set is in flight at once with no registers held.
//   * A cluster of CS = (G / HPC) * S CTAs serves one (sequence, query, KV
//     head).  CTA rank = hg * S + sh owns the HPC query heads of head group hg
//     and share sh of their candidates and kept leaves.  With S = 1 a level's
//     scores, top-k and kept list stay in the CTA; with S > 1 the S CTAs of a
//     head group store their scores into each other's shared memory
//     (distributed shared memory) and signal each other's "scores ready"
//     mbarrier.  HPC and S are chosen per launch so that the grid fills the
//     148 SMs.
//   * Warps are specialised.  Twelve chain warps walk the levels (score,
//     then one warp per head selects, writes the kept list and issues the
//     next level's key copies, then all fold the unselected summary values
//     while those copies fly) and then stream the kept leaves through a ring
//     of bulk-copy slots.  Three window warps attend the exact window, which
//     does not depend on the selection, through their own ring of bulk-copy
//     slots, concurrently with the chain; each CTA sends its window partial of
//     every head to that head's owner at the end.  One producer warp issues
//     the level values' and the later kept leaves' copies.
//   * Rows are read from shared memory with 16-byte (fp32) or 8-byte (bf16)
//     loads: a row is spread over d/8 lanes, each lane holding four
//     rotate-half pairs (j, j + d/2), so the RoPE rotation is local to the
//     lane.  Each lane slot keeps an online softmax state; states are merged
//     across slots, warps and finally the cluster (through distributed shared
//     memory) without any global scratch.
//   * Every wait on an mbarrier is bounded; on expiry the kernel sets
//     RECSA_DEVERR_WAIT_TIMEOUT in the tree header and runs to completion.
#include <cooperative_groups.h>
#include <cstdio>
#include <cstdlib>

#include "recsa_internal.cuh"
#include "rows.cuh"
#include "pool.cuh"

namespace cg = cooperative_groups;

namespace recsa {
namespace {

constexpr int kThreads = 512;

constexpr int kChainWarps = 12;
constexpr int kWinWarps = 3;
constexpr int kProducerWarp = kChainWarps + kWinWarps;   // issues the chain's copies
constexpr int kChainThreads = kChainWarps * 32;
constexpr int kRegSlots = 8;      // top-k candidates held in registers: 32 per slot
constexpr int kWinRing = 4;       // window ring slots
constexpr int kWinChunk = 24;     // window rows per ring slot
constexpr int kMaxCluster = 16;
constexpr int kMaxTokSlots = 4;   // kept-leaf ring slots per head
constexpr unsigned long long kWaitNs = 50000000ull;   // a wait gives up after 50 ms
constexpr size_t kSmemLimit = 227 * 1024;

// Named barriers (0 is __syncthreads).
constexpr int kBarChain = 1;      // the chain warps
constexpr int kBarWindow = 2;     // the window warps
constexpr int kBarHead0 = 3;      // + h: the chain warps of local head h

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

// ---------------------------------------------------------------------------
// PTX wrappers: mbarriers, bulk copies, cluster barriers, named barriers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned smem_addr(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* mb, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(mb)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
// Arrive once on mb and add `bytes` to the transaction count of its phase.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* mb, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(mb)),
               "r"(bytes)
               : "memory");
}
// Arrive once (release at cluster scope) on the mbarrier at the same offset
// in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* mb, int rank) {
  unsigned remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n"
               : "=r"(remote)
               : "r"(smem_addr(mb)), "r"(rank));
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(remote)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* mb, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(mb)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_test_wait(uint64_t* mb, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(mb)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of the given parity.  False when it did not
// complete within kWaitNs, or when an earlier wait of this thread expired
// (`expired` is then set, and later waits return at once so that the kernel
// runs to completion).
__device__ __forceinline__ bool mbar_wait(uint64_t* mb, unsigned parity, bool& expired) {
  if (expired) return false;
  if (mbar_test_wait(mb, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(mb, parity)) return true;
    if (global_ns() - t0 > kWaitNs) {
      expired = true;
      return false;
    }
  }
}
// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global memory into this CTA's shared memory, completing on mb.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         uint64_t* mb) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(mb))
      : "memory");
}
// Arrive once on mb (release at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t* mb) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(mb)) : "memory");
}
// Orders this thread's earlier shared-memory accesses (and those it has
// synchronised with) before later bulk copies into shared memory.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void fence_cluster() {
  asm volatile("fence.acq_rel.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");
}

// Online-softmax state (m, l, acc) of a lane slot merged with the state held by
// the lanes `o` apart (shuffles); every lane ends with the merged state.
__device__ __forceinline__ void merge_xor(float& m, float& l, float* acc, int o) {
  const float mo = __shfl_xor_sync(0xffffffffu, m, o);
  const float lo = __shfl_xor_sync(0xffffffffu, l, o);
  const float mn = fmaxf(m, mo);
  const float ra = (m == -INFINITY) ? 0.f : __expf(m - mn);
  const float rb = (mo == -INFINITY) ? 0.f : __expf(mo - mn);
  l = l * ra + lo * rb;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float ao = __shfl_xor_sync(0xffffffffu, acc[c], o);
    acc[c] = acc[c] * ra + ao * rb;
  }
  m = mn;
}

// Shared-memory plan of one CTA (byte offsets), the same on host and device.
struct Plan {
  unsigned mb, geo, qf, qtok, qlev, rrow, sc, agg, wsc, wwin, gsc, mrg, kept, tk, rmask, wbuf,
      kbuf, vbuf, total;
  int rows;         // summary rows per local head in kbuf and vbuf (one share of a level)
  unsigned kbytes;  // bytes of a level's keys in kbuf
  unsigned kreg;    // bytes before vbuf (the kept-leaf ring starts at kbuf and may run into vbuf)
};
template <typename T, int D, int G, int HPC>
__host__ __device__ __forceinline__ Plan make_plan(int cmax, int kmax, int S, int CS, int NRH,
                                                   int B, int levels, int HB) {
  constexpr unsigned RS = D + 2;
  Plan q;
  unsigned o = 0;
  q.mb = o;   o += 512;                                   // mbarriers
  q.geo = o;  o += (kMaxLevels + 2) * 16 + 16;            // per-level counts, top level
  q.qf = o;   o += G * D * 4;
  q.qtok = o; o += G * D * 4;
  q.qlev = o; o += unsigned(levels) * HPC * D * 4;        // query rotated per level
  q.rrow = o; o += unsigned(2 * levels + 3) * D * 4;      // RoPE table rows (cos, sin)
  q.sc = o;   o += 2 * HPC * unsigned(cmax) * 4;
  q.agg = o;  o += unsigned(cmax) * 4;                    // group scores (RECSA_MODE_GROUP)
  q.wsc = o;  o += kChainWarps * RS * 4;
  q.wwin = o; o += kWinWarps * G * RS * 4;
  q.gsc = o;  o += 2 * kChainWarps * 4;                   // group scores: per-warp (max, sum)
  q.mrg = o;  o += unsigned(CS) * HPC * RS * 4;
  q.kept = o; o += 2 * HPC * unsigned(kmax) * 4;
  o = (o + 7u) & ~7u;
  q.tk = o;   o += HPC * 32 * 8;                          // selection scratch (key, index)
  o = (o + 15u) & ~15u;
  q.rmask = o; o += HPC * 32 * 4;
  o = (o + 127u) & ~127u;
  q.wbuf = o; o += kWinRing * 2 * kWinChunk * D * unsigned(sizeof(T));
  o = (o + 127u) & ~127u;
  q.kbuf = o;
  q.rows = (cmax + S - 1) / S;
  q.kbytes = unsigned(HB) * unsigned(q.rows) * D * 4;   // HB heads' level rows
  // with one buffer head, at least two kept-leaf slots before vbuf, so that
  // the first leaves can be copied as soon as level 1 is selected (the rest
  // once its values are folded)
  const unsigned slot = 2 * unsigned(B) * D * unsigned(sizeof(T));
  const unsigned early = HB == 1 ? unsigned(NRH < 2 ? NRH : 2) * slot : 0u;
  q.kreg = q.kbytes > early ? q.kbytes : early;
  q.vbuf = o + q.kreg;
  const unsigned toks = unsigned(HB) * unsigned(NRH) * slot;
  o += q.kreg + q.kbytes > toks ? q.kreg + q.kbytes : toks;
  q.total = o;
  return q;
}

// Pooling after the fused step's append (one warp): the leaf the new token
// completes, then every ancestor it completes in turn.  Out of line: it runs
// in one CTA per (sequence, KV head) at the end of the step.
template <typename T, int D>
__device__ __noinline__ void pool_appended(const Params& p, const T* K, const T* V, const void* tree,
                                           const float* r, int64_t kvbase, int64_t t, int64_t seq,
                                           int g, int lane) {
  constexpr int N = D / 32;
  float rl[N], key[N], val[N];
  load_r<N>(r, lane, rl);
  int64_t j = (t + 1) / p.B - 1;
  const int64_t row0 = (kvbase + j * p.B) * D;
  pool_rows<T, N>(K + row0, V + row0, p.B, D, rl, p.inv_sqrt_d, lane, key, val);
  RowIO<float, N>::store(level_keys(p, const_cast<void*>(tree), 1, seq, g) + j * D, lane, key);
  RowIO<float, N>::store(level_vals(p, const_cast<void*>(tree), 1, seq, g) + j * D, lane, val);
  for (int lev = 2; lev <= p.lay.levels && (j + 1) % p.b == 0; ++lev) {
    j = (j + 1) / p.b - 1;
    __syncwarp();
    const float* ck = level_keys(p, const_cast<void*>(tree), lev - 1, seq, g) + j * p.b * D;
    const float* cv = level_vals(p, const_cast<void*>(tree), lev - 1, seq, g) + j * p.b * D;
    pool_rows<float, N>(ck, cv, p.b, D, rl, p.inv_sqrt_d, lane, key, val);
    RowIO<float, N>::store(level_keys(p, const_cast<void*>(tree), lev, seq, g) + j * D, lane, key);
    RowIO<float, N>::store(level_vals(p, const_cast<void*>(tree), lev, seq, g) + j * D, lane, val);
  }
}

template <typename T, int D, int G, int HPC>
__global__ void __launch_bounds__(kThreads, 1)
decode_cluster_kernel(const __grid_constant__ Params p, const T* __restrict__ Q, const T* __restrict__ K,
                      const T* __restrict__ V, const void* __restrict__ tree,
                      const int64_t* __restrict__ len_dev, int n_q, T* __restrict__ O,
                      int32_t* __restrict__ trace, int cmax, int kmax, int S, int NRH,
                      StepArgs st) {
  constexpr int HALF = D / 2, LPR = HALF / 4, SPW = 32 / LPR;
  constexpr int WPH = kChainWarps / HPC, HSLOT = WPH * SPW;
  constexpr int WSL = kWinWarps * SPW;                 // window lane slots
  constexpr int RS = D + 2;                            // merge row: acc[D], m, l
  static_assert(kChainWarps % HPC == 0, "chain warps split evenly over the heads");
  static_assert(kWinChunk % WSL == 0, "window slots advance evenly across chunks");
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = int(cluster.num_blocks());
  const int rank = int(cluster.block_rank());
  const int hg = rank / S, sh = rank % S;              // head group, candidate share
  const int qi = blockIdx.y;
  const int64_t seq = blockIdx.z / p.hkv;
  const int g = int(blockIdx.z % p.hkv);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR;
  const int j0 = 4 * sub;

  // RECSA_MODE_GROUP: the G heads share one selection, hence one copy of a
  // level's candidate rows and one ring of kept leaves (HB = 1 buffer head).
  // (only launched with every head of the group in the CTA: HPC == G)
  const bool grp = HPC == G && p.mode == RECSA_MODE_GROUP;
  const int HB = grp ? 1 : HPC;
  const Plan pl = make_plan<T, D, G, HPC>(cmax, kmax, S, CS, NRH, p.B, p.lay.levels, HB);
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* mb_lev = reinterpret_cast<uint64_t*>(smem + pl.mb);   // level keys arrived
  uint64_t* mb_val = mb_lev + 1;                                   // level values arrived
  uint64_t* mb_ready = mb_lev + 2;             // [2] head group's scores by level parity (S > 1)
  uint64_t* mb_kept = mb_lev + 4;              // chain -> producer: a level's kept list is ready
  uint64_t* mb_folded = mb_lev + 5;            // chain -> producer: a level's values are folded
  uint64_t* mb_win = mb_lev + 6;                                   // [kWinRing]
  uint64_t* mb_tok = mb_win + kWinRing;                            // [HPC][NRH] leaf arrived
  uint64_t* mb_empty = mb_tok + HPC * NRH;                         // [HPC][NRH] slot consumed
  uint64_t* mb_never = mb_lev + 63;   // no thread ever arrives (expiry test, last mbarrier slot)
  float* qf = reinterpret_cast<float*>(smem + pl.qf);       // [G][D] raw query
  float* qtok = reinterpret_cast<float*>(smem + pl.qtok);   // [G][D] rotated to n0 - 1
  float* qlev = reinterpret_cast<float*>(smem + pl.qlev);   // [levels][HPC][D] rotated to c_l
  // RoPE table rows: [l - 1] = R(lo_l) (first candidate of this share at level
  // l), [levels] = R(sh * B), [levels + 1] = R(S * B), [levels + 1 + l] =
  // R(c_l) (the query's index at level l), [2 levels + 2] = R(n0 - 1)
  float* rrow = reinterpret_cast<float*>(smem + pl.rrow);
  float* sc = reinterpret_cast<float*>(smem + pl.sc);       // [2][HPC][cmax] scores
  float* agg = reinterpret_cast<float*>(smem + pl.agg);     // [cmax] group scores
  float* wsc = reinterpret_cast<float*>(smem + pl.wsc);     // [kChainWarps][RS]
  float* wwin = reinterpret_cast<float*>(smem + pl.wwin);   // [kWinWarps][G][RS]
  float* gsc = reinterpret_cast<float*>(smem + pl.gsc);     // [kChainWarps][2]
  float* mrg = reinterpret_cast<float*>(smem + pl.mrg);     // [CS][HPC][RS] received
  int* kept = reinterpret_cast<int*>(smem + pl.kept);       // [2][HPC][kmax]
  uint2* tkl = reinterpret_cast<uint2*>(smem + pl.tk);     // [HPC][32] selection scratch
  unsigned* rmask = reinterpret_cast<unsigned*>(smem + pl.rmask);   // [HPC][32] kept bits
  T* wbuf = reinterpret_cast<T*>(smem + pl.wbuf);           // [kWinRing][2][kWinChunk][D]
  float* kbuf = reinterpret_cast<float*>(smem + pl.kbuf);   // [HB][rows][D] level keys
  float* vbuf = reinterpret_cast<float*>(smem + pl.vbuf);   // [HB][rows][D] level values
  T* tbuf = reinterpret_cast<T*>(smem + pl.kbuf);           // [HB][NRH][2][B][D] kept leaves

  // The query and the chain slots' RoPE steps do not depend on the sequence
  // length: their loads are issued first, beside the length's.
  static_assert(G * D <= kThreads, "one query element per thread");
  const int64_t qrow = ((seq * n_q + qi) * p.hq + int64_t(g) * G) * D;
  const float qpre = tid < G * D ? load_elem(Q, qrow + tid, p.dtype) : 0.f;
  const float2* rope = rope_table(p, tree);
  const int rmax = p.lay.rope_rows - 1;
  // Chain warps [h * WPH, (h + 1) * WPH) serve local query head h (global
  // head hg * HPC + h); hs is the lane slot's index within the head's warps.
  const int hw = warp / WPH;
  const int hb = grp ? 0 : hw;   // its buffer head
  const int hs = (warp % WPH) * SPW + lane / LPR;
  // RoPE of the slot's first row and of its row step, for the recurrences
  float cs_hs[8], cs_st[8];
  if (p.rope && warp < kChainWarps) {
    load_cs(rope, min(hs, rmax), HALF, j0, cs_hs);
    load_cs(rope, min(HSLOT, rmax), HALF, j0, cs_st);
  }
  // Fused step: the new token is appended at len (this kernel writes it and
  // pools what it completes), and the query sits on it.  A full sequence is
  // flagged and decoded without the append, as recsa_append would leave it.
  const int64_t len0 = len_dev[seq];
  const bool do_append = st.fuse && len0 >= 0 && len0 < p.cap;
  const int64_t t = do_append ? len0 : len0 - 1;
  const T* knew = reinterpret_cast<const T*>(st.k_new) + (seq * p.hkv + g) * D;
  const T* vnew = reinterpret_cast<const T*>(st.v_new) + (seq * p.hkv + g) * D;
  const bool empty = t < 0 || t >= p.cap;   // uniform over the cluster
  const int64_t s0 = t + 1 - p.W > 0 ? t + 1 - p.W : 0;
  const int64_t a = empty ? 0 : (s0 <= 0x7fffffff ? int64_t(div_B(p, int(s0))) : s0 / p.B);
  // Per-level counts, the same for every head, computed once into shared
  // memory (indexed by level at run time, so registers cannot hold them):
  // vis[l] = complete nodes of level l visible to the query (before the
  // window), cnt_c[l] / cnt_k[l] = candidates / kept at level l, and the top
  // level with a visible node.
  int64_t* vis = reinterpret_cast<int64_t*>(smem + pl.geo);
  int* cnt_c = reinterpret_cast<int*>(vis + kMaxLevels + 2);
  int* cnt_k = cnt_c + kMaxLevels + 2;
  int* top_s = cnt_k + kMaxLevels + 2;
  if (tid == 0) {
    int tp = 0;
    int64_t v = a;
    for (int lev = 1; lev <= p.lay.levels; ++lev) {
      vis[lev] = v;
      if (v == 0) break;
      tp = lev;
      v = v <= 0x7fffffff ? int64_t(div_b(p, int(v))) : v / p.b;
    }
    int kup = 0;
    for (int lev = tp; lev >= 1; --lev) {
      const int64_t vup = lev < tp ? vis[lev + 1] : 0;
      cnt_c[lev] = p.b * kup + int(vis[lev] - p.b * vup);
      cnt_k[lev] = cnt_c[lev] < p.k ? cnt_c[lev] : p.k;
      kup = cnt_k[lev];
    }
    *top_s = tp;
  }
  const int64_t n_win = empty ? 0 : t + 1 - a * p.B;
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  const float inv_sqrt_d = p.inv_sqrt_d;
  const int tstride = kTraceHead + kMaxLevels * p.k;
  unsigned* errw = tree_error_word(const_cast<void*>(tree));

  // This CTA's share [lo, hi) of tot items split over the head group's S CTAs.
  auto share = [&](int tot, int& lo, int& hi) {
    const int ch = (tot + S - 1) / S;
    lo = min(tot, sh * ch);
    hi = min(tot, lo + ch);
  };
  // Window share of this CTA (rows of the whole cluster split by rank).
  int w_lo = 0, w_hi = 0;
  {
    const int nw = int(n_win), ch = (nw + CS - 1) / CS;
    w_lo = min(nw, rank * ch);
    w_hi = min(nw, w_lo + ch);
  }
  const int nwr = w_hi - w_lo;
  const int nwch = (nwr + kWinChunk - 1) / kWinChunk;

  if (tid == 0) {
    mbar_init(mb_lev, unsigned(HB));   // one arrival per buffer head (its selection warp)
    mbar_init(mb_val, 1);
    mbar_init(mb_kept, HPC);
    mbar_init(mb_folded, 1);
    mbar_init(mb_never, 1);
    mbar_init(mb_ready, unsigned(S));
    mbar_init(mb_ready + 1, unsigned(S));
    for (int i = 0; i < kWinRing; ++i) mbar_init(mb_win + i, 1);
    for (int i = 0; i < HPC * NRH; ++i) {
      mbar_init(mb_tok + i, 1);
      mbar_init(mb_empty + i, grp ? unsigned(HPC) : 1u);   // a shared slot: every head frees it
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (CS > 1) cluster_arrive_relaxed();   // waited on before the first remote access
  const int top = *top_s;
  const int nleaf = top > 0 ? cnt_k[1] : 0;
  const int64_t n0 = int64_t(nleaf) * p.B + n_win;
  // kept leaves of this share (leaf ranks sh, sh + S, ...)
  const int ntok = nleaf > sh ? (nleaf - sh + S - 1) / S : 0;

  // ---- producers (bulk copies) ----------------------------------------------
  // Node id of candidate i of local head h at level lev (kept list of lev + 1).
  auto cand_node = [&](int lev, int h, int i) -> int {
    const int kup = lev < top ? cnt_k[lev + 1] : 0;
    const int vup = lev < top ? int(vis[lev + 1]) : 0;
    if (i < p.b * kup)
      return kept[((lev + 1) & 1) * HPC * kmax + h * kmax + div_b(p, i)] * p.b + mod_b(p, i);
    return p.b * vup + (i - p.b * kup);
  };
  // Keys (or values) of level lev (this CTA's share [lo, hi) of the candidate
  // list of each local head) into kbuf (vbuf) in candidate order, completing
  // on mb_lev (mb_val).  Run by the whole producer warp: lane 0 arms the
  // barrier, the lanes copy one run each (the children of a kept node of
  // level lev + 1, or the orphans; the top level is one run).  Below the top
  // level the keys are issued by the selection warps instead (one arrival
  // per buffer head on mb_lev), so the top level's keys arrive HB times too.
  auto issue_level = [&](int lev, bool values) {
    const int c = cnt_c[lev];
    int lo, hi;
    share(c, lo, hi);
    const unsigned rb = D * 4;
    uint64_t* mb = values ? mb_val : mb_lev;
    float* dst = values ? vbuf : kbuf;
    if (lane == 0) {
      mbar_expect_tx(mb, unsigned(HB) * unsigned(hi - lo) * rb);
      if (!values)
        for (int n = 1; n < HB; ++n) mbar_arrive(mb);
    }
    __syncwarp();
    if (hi <= lo) return;
    const float* src = values ? level_vals(p, const_cast<void*>(tree), lev, seq, g)
                              : level_keys(p, const_cast<void*>(tree), lev, seq, g);
    const int kup = lev < top ? cnt_k[lev + 1] : 0;
    const int nch = p.b * kup;
    const int orph0 = lev < top ? p.b * int(vis[lev + 1]) : 0;   // first orphan node
    const int* keptu = kept + ((lev + 1) & 1) * HPC * kmax;
    const int nrun = kup + 1;
    for (int x = lane; x < HB * nrun; x += 32) {
      const int h = x / nrun, r = x % nrun;
      int c0, c1, node0;
      if (r < kup) {
        c0 = r * p.b;
        c1 = c0 + p.b;
        node0 = keptu[h * kmax + r] * p.b;
      } else {
        c0 = nch;
        c1 = c;
        node0 = orph0;
      }
      const int a0 = max(c0, lo), a1 = min(c1, hi);
      if (a1 > a0)
        bulk_g2s(dst + (size_t(h) * pl.rows + (a0 - lo)) * D,
                 src + int64_t(node0 + (a0 - c0)) * D, unsigned(a1 - a0) * rb, mb);
    }
  };
  // Window chunk ch (rows [ch * kWinChunk, ...) of this CTA's window share)
  // into ring slot ch % kWinRing; the new token's row comes from k_new/v_new.
  auto issue_win = [&](int ch) {
    const int slot = ch % kWinRing;
    const int r0 = ch * kWinChunk, r1 = min(nwr, r0 + kWinChunk);
    const int nrow = r1 - r0;
    const int64_t p0 = a * p.B + w_lo + r0;            // position of the first row
    const bool newrow = do_append && p0 + nrow - 1 == t;
    const int nk = newrow ? nrow - 1 : nrow;
    const unsigned eb = D * unsigned(sizeof(T));
    uint64_t* mb = mb_win + slot;
    mbar_expect_tx(mb, 2u * unsigned(nrow) * eb);
    T* dK = wbuf + size_t(slot) * 2 * kWinChunk * D;
    T* dV = dK + size_t(kWinChunk) * D;
    if (nk > 0) {
      bulk_g2s(dK, K + (kvbase + p0) * D, unsigned(nk) * eb, mb);
      bulk_g2s(dV, V + (kvbase + p0) * D, unsigned(nk) * eb, mb);
    }
    if (newrow) {
      bulk_g2s(dK + size_t(nk) * D, knew, eb, mb);
      bulk_g2s(dV + size_t(nk) * D, vnew, eb, mb);
    }
  };
  // Kept leaf j of buffer head h's share (leaf rank sh + j * S, leaf `node`)
  // into its ring slot: B rows of K, then B rows of V.
  auto issue_tok_node = [&](int h, int j, int node) {
    const int slot = j % NRH;
    const unsigned lb = unsigned(p.B) * D * unsigned(sizeof(T));
    uint64_t* mb = mb_tok + h * NRH + slot;
    mbar_expect_tx(mb, 2u * lb);
    T* dK = tbuf + (size_t(h) * NRH + slot) * 2 * p.B * D;
    bulk_g2s(dK, K + (kvbase + int64_t(node) * p.B) * D, lb, mb);
    bulk_g2s(dK + size_t(p.B) * D, V + (kvbase + int64_t(node) * p.B) * D, lb, mb);
  };
  auto issue_tok = [&](int h, int j) {
    issue_tok_node(h, j, kept[1 * HPC * kmax + h * kmax + sh + j * S]);   // level 1's list
  };


  // First copies: the top level's keys and values (the producer warp), before
  // the query is loaded.
  if (warp == kProducerWarp && top > 0) {
    issue_level(top, false);
    issue_level(top, true);
  }
  // The query and the RoPE table rows the kernel needs (loaded together: one
  // memory round trip), then the query rotated to every level's index.
  if (tid < G * D) qf[tid] = empty ? 0.f : qpre;
  if (p.rope) {
    const int lv = p.lay.levels;
    for (int x = tid; x < (2 * lv + 3) * HALF; x += kThreads) {
      const int r = x / HALF, j = x % HALF;
      int64_t idx = -1;
      if (r < lv) {
        if (r < top) {
          int lo, hi;
          share(cnt_c[r + 1], lo, hi);
          idx = lo;
        }
      } else if (r == lv) {
        idx = int64_t(sh) * p.B;
      } else if (r == lv + 1) {
        idx = int64_t(S) * p.B;
      } else if (r < 2 * lv + 2) {
        if (r - lv - 1 <= top) idx = cnt_c[r - lv - 1];
      } else {
        idx = n0 - 1 > 0 ? n0 - 1 : 0;
      }
      if (idx < 0) continue;
      const float2 cs = rope[min(idx, int64_t(rmax)) * HALF + j];
      rrow[r * D + 2 * j] = cs.x;
      rrow[r * D + 2 * j + 1] = cs.y;
    }
  }
  for (int x = tid; x < kWinWarps * G * RS; x += kThreads)
    wwin[x] = (x % RS == D) ? -INFINITY : 0.f;
  __syncthreads();
  // qf rows [h0, h0 + nh) rotated by table row r of rrow into dst.
  auto rotate_q = [&](float* dst, int h0, int nh, int r) {
    for (int x = tid; x < nh * HALF; x += kThreads) {
      const int h = x / HALF, j = x % HALF;
      const float x1 = qf[(h0 + h) * D + j], x2 = qf[(h0 + h) * D + j + HALF];
      if (p.rope) {
        const float c = rrow[r * D + 2 * j], sn = rrow[r * D + 2 * j + 1];
        dst[h * D + j] = x1 * c - x2 * sn;
        dst[h * D + j + HALF] = x2 * c + x1 * sn;
      } else {
        dst[h * D + j] = x1;
        dst[h * D + j + HALF] = x2;
      }
    }
  };
  if (!empty) rotate_q(qtok, 0, G, 2 * p.lay.levels + 2);
  for (int lev = 1; lev <= top; ++lev)
    rotate_q(qlev + (lev - 1) * HPC * D, hg * HPC, HPC, p.lay.levels + 1 + lev);
  __syncthreads();
  if (CS > 1) cluster_wait();
  bool timed_out = false;   // a bounded wait of this thread expired

  // ---- window warps ---------------------------------------------------------
  // Rows of this CTA's window share, scored once for all G heads of the group
  // (each lane slot keeps one online softmax per head), chunk by chunk through
  // the ring; the warp's per-head partials end in wwin.
  auto window_warps = [&]() {
    const int wl = warp - kChainWarps;
    const int gsl = wl * SPW + lane / LPR;
    // the first chunks of the ring (issued here, off the prologue's barriers)
    if (warp == kChainWarps && lane < kWinRing && lane < nwch) issue_win(lane);
    float mW[G], lW[G], accW[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mW[h] = -INFINITY;
      lW[h] = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) accW[h][c] = 0.f;
    }
    // a slot's rows are gsl, gsl + WSL, ... across all chunks: its RoPE
    // index grows by WSL per row, so its (cos, sin) advance by a fixed step
    const int widx0 = nleaf * p.B + w_lo;
    float qr[G][8];   // the query of every head, rotated to n0 - 1
#pragma unroll
    for (int h = 0; h < G; ++h) lds_pairs(qtok + h * D, j0, HALF, qr[h]);
    float csc[8], cstep[8];
    const bool recur = WSL <= rmax;
    if (p.rope && recur && nwch > 0) {
      load_cs(rope, min(widx0 + gsl, rmax), HALF, j0, csc);
      load_cs(rope, WSL, HALF, j0, cstep);
    }
    for (int ch = 0; ch < nwch; ++ch) {
      const int slot = ch % kWinRing;
      mbar_wait(mb_win + slot, unsigned(ch / kWinRing) & 1u, timed_out);
      const T* cK = wbuf + size_t(slot) * 2 * kWinChunk * D;
      const T* cV = cK + size_t(kWinChunk) * D;
#pragma unroll 1
      for (int e = gsl; e < kWinChunk; e += WSL) {
        const int r = ch * kWinChunk + e;
        const bool on = r < nwr;
        float xk[8], xv[8];
        SharedPairs<T, HALF>::load(cK + size_t(e) * D, j0, xk);
        SharedPairs<T, HALF>::load(cV + size_t(e) * D, j0, xv);
        if (p.rope) {
          if (!recur) load_cs(rope, min(widx0 + r, rmax), HALF, j0, csc);
          rotate8(xk, csc);
          if (recur) advance_cs(csc, cstep);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float s = slot_sum<LPR>(dot8(qr[h], xk)) * inv_sqrt_d;
          if (on) fold8(mW[h], lW[h], accW[h], s, xv);
        }
      }
      named_sync(kBarWindow, kWinWarps * 32);
      if (warp == kChainWarps && lane == 0 && ch + kWinRing < nwch) {
        fence_proxy_async();
        issue_win(ch + kWinRing);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) merge_xor(mW[h], lW[h], accW[h], o);
      if (lane < LPR) {
        float* w = wwin + (wl * G + h) * RS;
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

  // ---- chain warps ----------------------------------------------------------
  // Every lane slot of a chain warp keeps one online-softmax state of its head.
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;


  // Scores of this CTA's share of level lev's candidates (keys in kbuf) for
  // head hw, two rows per slot at a time; with S > 1 each score is stored
  // into every CTA of the group.  The score of candidate i is
  // <R(c) q, R(i) k> = <R(c - i) q, k>, so the query (rotated to c in qlev)
  // is turned back by the candidate's index instead of rotating every key: a
  // slot's rows are lo + hs + j * HSLOT, so its query starts at
  // R(-(lo + hs)) qlev and turns by R(-HSLOT) per row.
  auto score_level = [&](int lev) {
    int lo, hi;
    share(cnt_c[lev], lo, hi);
    const int nr = hi - lo;
    const float* kb = kbuf + size_t(hb) * pl.rows * D;
    float* scK = sc + (lev & 1) * HPC * cmax + hw * cmax + lo;
    float q0[8], st2[8];
    lds_pairs(qlev + ((lev - 1) * HPC + hw) * D, j0, HALF, q0);
    if (p.rope) {
      float seed[8], t[8];
      if (S == 1) {
#pragma unroll
        for (int c = 0; c < 8; ++c) seed[c] = cs_hs[c];
      } else {
        float r[8];
        lds_cs8(rrow + (lev - 1) * D, j0, r);
        cmul8(seed, r, cs_hs);
      }
      rot_neg8(t, q0, seed);
#pragma unroll
      for (int c = 0; c < 8; ++c) q0[c] = t[c];
      cmul8(st2, cs_st, cs_st);
    }
    for (int e = hs; e - hs < nr; e += 2 * HSLOT) {
      const int e1 = e + HSLOT;
      const bool on0 = e < nr, on1 = e1 < nr;
      float x0[8], x1[8], q1[8];
      SharedPairs<float, HALF>::load(kb + size_t(on0 ? e : 0) * D, j0, x0);
      SharedPairs<float, HALF>::load(kb + size_t(on1 ? e1 : 0) * D, j0, x1);
      if (p.rope) {
        rot_neg8(q1, q0, cs_st);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) q1[c] = q0[c];
      }
      float s0 = dot8(q0, x0), s1 = dot8(q1, x1);
      if (p.rope) {
        float t[8];
        rot_neg8(t, q0, st2);
#pragma unroll
        for (int c = 0; c < 8; ++c) q0[c] = t[c];
      }
      slot_sum2<LPR>(s0, s1);
      s0 *= inv_sqrt_d;
      s1 *= inv_sqrt_d;
      if (S == 1) {
        if (sub == 0) {
          if (on0) scK[e] = s0;
          if (on1) scK[e1] = s1;
        }
      } else {
        if (sub < S) {
          if (on0) *cluster.map_shared_rank(scK + e, hg * S + sub) = s0;
          if (on1) *cluster.map_shared_rank(scK + e1, hg * S + sub) = s1;
        }
        if (sub + LPR < S) {
          if (on0) *cluster.map_shared_rank(scK + e, hg * S + sub + LPR) = s0;
          if (on1) *cluster.map_shared_rank(scK + e1, hg * S + sub + LPR) = s1;
        }
      }
    }
  };

  // Values of this CTA's share of level lev's unselected candidates (head
  // hw, rows in vbuf in candidate order), folded two rows at a time.
  auto fold_values = [&](int lev) {
    int lo, hi;
    share(cnt_c[lev], lo, hi);
    const int nr = hi - lo;
    const float* vb = vbuf + size_t(hb) * pl.rows * D;
    const float* scV = sc + (lev & 1) * HPC * cmax + hw * cmax + lo;
    const unsigned* msk = rmask + hw * 32;
    auto kept_bit = [&](int i) { return (msk[i >> 5] >> (i & 31)) & 1u; };
    for (int e = hs; e < nr; e += 2 * HSLOT) {
      const int e1 = e + HSLOT;
      const bool on0 = !kept_bit(lo + e), on1 = e1 < nr && !kept_bit(lo + e1);
      float x0[8], x1[8];
      SharedPairs<float, HALF>::load(vb + size_t(e) * D, j0, x0);
      SharedPairs<float, HALF>::load(vb + size_t(on1 ? e1 : e) * D, j0, x1);
      fold2(m, l, acc, scV[e], on0, x0, on1 ? scV[e1] : 0.f, on1, x1);
    }
  };


  // Slot s of local head h lies inside kbuf (free once the level-1 keys are
  // scored) rather than reaching into vbuf (free once the level-1 values are
  // folded).
  auto early_slot = [&](int h, int s) {
    const size_t sb = size_t(2) * p.B * D * sizeof(T);
    return (size_t(h) * NRH + s + 1) * sb <= pl.kreg;
  };
  // RECSA_MODE_GROUP (every head of the group in the CTA, HPC == G): the
  // group score of candidate i is the sum over the heads of its softmax
  // probability among the level's candidates, computed by all chain threads.
  // Chain warp w takes head w % G and a strided part of the candidates: an
  // online (max, sum of exp) pass, reduced over the warp into gsc; then each
  // thread combines the parts of every head for its candidates.  Ends with a
  // chain barrier (agg complete).
  auto group_scores = [&](int lev) {
    constexpr int NP = kChainWarps / G;   // parts per head
    static_assert(kChainWarps % G == 0, "chain warps split evenly over the heads");
    const int c = cnt_c[lev], par = lev & 1;
    const float* scl = sc + par * HPC * cmax;
    {
      const int h = warp % G, part = warp / G;
      const float* rw = scl + h * cmax;
      float mx = -INFINITY, sm = 0.f;
      for (int i = part * 32 + lane; i < c; i += NP * 32) {
        const float v = rw[i];
        if (v > mx) {
          sm = (mx == -INFINITY ? 0.f : sm * expf(mx - v)) + 1.f;
          mx = v;
        } else {
          sm += expf(v - mx);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, mx, o);
        const float so = __shfl_xor_sync(0xffffffffu, sm, o);
        const float mn = fmaxf(mx, mo);
        sm = (mx == -INFINITY ? 0.f : sm * expf(mx - mn)) + (mo == -INFINITY ? 0.f : so * expf(mo - mn));
        mx = mn;
      }
      if (lane == 0) {
        gsc[2 * warp] = mx;
        gsc[2 * warp + 1] = sm;
      }
    }
    named_sync(kBarChain, kChainThreads);
    float mh[G], zh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < NP; ++q) mx = fmaxf(mx, gsc[2 * (q * G + h)]);
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        const float mq = gsc[2 * (q * G + h)];
        if (mq != -INFINITY) z += gsc[2 * (q * G + h) + 1] * expf(mq - mx);
      }
      mh[h] = mx;
      zh[h] = z;
    }
    for (int i = tid; i < c; i += kChainThreads) {
      float a_ = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) a_ += expf(scl[h * cmax + i] - mh[h]) / zh[h];
      agg[i] = a_;
    }
    named_sync(kBarChain, kChainThreads);
  };

  // Selection of level lev for local head h = 3 - warp (warps 4 - HPC .. 3,
  // one per head) over the head's full score table; with S > 1 every CTA of
  // the head group runs the same selection on the same scores.
  // RECSA_MODE_GROUP (all G heads in the CTA): head 0's warp selects once for
  // the group on the group scores -- the sum over the heads of each
  // candidate's softmax probability among the level's candidates -- and
  // hands the same selection to every head.
  //   Candidates are ranked by order-preserving keys (0 = none), ties to the
  // lower index.  Lane l holds the keys of candidates l, l + 32, ... (the
  // first 32 * kRegSlots in registers, the rest read from shared memory).
  //   1. thr = the kap-th largest of the 32 lane maxima: at least kap
  //      candidates have a key >= thr, so the top kap are among them.
  //   2. The candidates with key >= thr (usually a few more than kap) are listed
  //      in the warp's scratch and ranked against each other by shuffles.
  //   (With more than 32 of them -- ties at the threshold -- or kap > 32, kap
  //   rounds of a warp arg-max pick the top kap instead.)
  // The kept bits land in rmask (bit l of word s = candidate 32 s + l); from
  // them the warp writes the kept list in index order (and the trace), and
  // then issues the copies that depend on it straight away: the next level's
  // key runs of this buffer head (one run per kept node, plus the orphans),
  // or, at level 1, the kept leaves whose ring slots lie in kbuf.
  auto select_level = [&](int lev) {
    const int c = cnt_c[lev], kap = cnt_k[lev];
    const int par = lev & 1;
    const int h = 3 - warp;
    if (grp && h != 0) return;
    const float* row = sc + par * HPC * cmax + h * cmax;
    if (grp) row = agg;   // the group scores (group_scores, all chain warps)
    const int ns = (c + 31) >> 5;
    const unsigned full = 0xffffffffu, lt = (1u << lane) - 1u;
    unsigned word = 0;   // lane s < ns: the kept bits of candidates 32 s .. 32 s + 31
    if (kap >= c) {
      if (lane < ns) word = (lane == ns - 1 && (c & 31)) ? (1u << (c & 31)) - 1u : full;
    } else {
      unsigned key[kRegSlots];
      unsigned lm = 0;
#pragma unroll
      for (int s = 0; s < kRegSlots; ++s) {
        const int i = s * 32 + lane;
        key[s] = i < c ? order_key(row[i]) : 0u;
        lm = max(lm, key[s]);
      }
      for (int s = kRegSlots; s < ns; ++s) {
        const int i = s * 32 + lane;
        if (i < c) lm = max(lm, order_key(row[i]));
      }
      bool fast = kap <= 32;
      unsigned thr = 1;
      if (fast) {
        int rk = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const unsigned o = __shfl_sync(full, lm, j);
          rk += (o > lm) | ((o == lm) & (j < lane));
        }
        const unsigned who = __ballot_sync(full, rk == kap - 1);
        thr = max(1u, __shfl_sync(full, lm, __ffs(who) - 1));
      }
      int cnt = 0;
#pragma unroll
      for (int s = 0; s < kRegSlots; ++s) cnt += key[s] >= thr;
      for (int s = kRegSlots; s < ns; ++s) {
        const int i = s * 32 + lane;
        if (i < c && order_key(row[i]) >= thr) ++cnt;
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(full, incl, o);
        if (lane >= o) incl += v;
      }
      const int nc = __shfl_sync(full, incl, 31);
      fast = fast && nc <= 32;
      if (fast) {
        uint2* tk = tkl + h * 32;
        int pos = incl - cnt;
#pragma unroll
        for (int s = 0; s < kRegSlots; ++s)
          if (key[s] >= thr) tk[pos++] = make_uint2(key[s], unsigned(s * 32 + lane));
        for (int s = kRegSlots; s < ns; ++s) {
          const int i = s * 32 + lane;
          if (i < c) {
            const unsigned kk = order_key(row[i]);
            if (kk >= thr) tk[pos++] = make_uint2(kk, unsigned(i));
          }
        }
        __syncwarp();
        const uint2 me = lane < nc ? tk[lane] : make_uint2(0u, 0u);
        int r = 0;
        for (int j = 0; j < nc; ++j) {
          const unsigned ok = __shfl_sync(full, me.x, j), oi = __shfl_sync(full, me.y, j);
          r += (ok > me.x) | ((ok == me.x) & (oi < me.y));
        }
        const bool kp = lane < nc && r < kap;
        for (int s = 0; s < ns; ++s) {
          const unsigned R =
              __reduce_or_sync(full, (kp && int(me.y >> 5) == s) ? 1u << (me.y & 31u) : 0u);
          if (lane == s) word = R;
        }
        __syncwarp();
      } else {
        unsigned taken = 0;
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
          const unsigned M = __reduce_max_sync(full, bk);
          unsigned who = __ballot_sync(full, bk == M);
          if (__popc(who) > 1) {
            const unsigned I =
                __reduce_min_sync(full, bk == M ? unsigned(bs * 32 + lane) : 0xffffffffu);
            who = 1u << (I & 31u);
          }
          if ((who >> lane) & 1u) {
            taken |= 1u << bs;
#pragma unroll
            for (int s = 0; s < kRegSlots; ++s)
              if (s == bs) key[s] = 0u;
          }
        }
        for (int s = 0; s < ns; ++s) {
          const unsigned R = __ballot_sync(full, (taken >> s) & 1u);
          if (lane == s) word = R;
        }
      }
    }
    if (lane < ns) {
      if (grp) {
#pragma unroll
        for (int hh = 0; hh < HPC; ++hh) rmask[hh * 32 + lane] = word;
      } else {
        rmask[h * 32 + lane] = word;
      }
    }
    // The kept list in index order, the trace, and the copies it unlocks.
    const int nxt = lev - 1;
    int lo2 = 0, hi2 = 0;
    if (nxt >= 1) share(cnt_c[nxt], lo2, hi2);
    const unsigned rb = D * 4;
    float* kdst = kbuf + size_t(h) * pl.rows * D;   // buffer head h (0 in group mode)
    const float* ksrc = nxt >= 1 ? level_keys(p, const_cast<void*>(tree), nxt, seq, g) : nullptr;
    fence_proxy_async();   // kbuf was read by the scoring threads (before the level barrier)
    if (nxt >= 1 && lane == 0) mbar_expect_tx(mb_lev, unsigned(hi2 - lo2) * rb);
    __syncwarp();
    int base = 0;
    for (int s = 0; s < ns; ++s) {
      const unsigned wv = __shfl_sync(full, word, s);
      if ((wv >> lane) & 1u) {
        const int pos = base + __popc(wv & lt);
        const int node = cand_node(lev, h, s * 32 + lane);
        for (int hh = grp ? 0 : h; hh < (grp ? HPC : h + 1); ++hh) {
          kept[par * HPC * kmax + hh * kmax + pos] = node;
          if (trace && sh == 0) {
            const int64_t rec =
                ((seq * n_q + qi) * p.hq + int64_t(g) * G + hg * HPC + hh) * tstride;
            trace[rec + kTraceHead + (lev - 1) * p.k + pos] = node;
          }
        }
        if (nxt >= 1) {
          const int c0 = pos * p.b, a0 = max(c0, lo2), a1 = min(c0 + p.b, hi2);
          if (a1 > a0)
            bulk_g2s(kdst + size_t(a0 - lo2) * D, ksrc + (int64_t(node) * p.b + (a0 - c0)) * D,
                     unsigned(a1 - a0) * rb, mb_lev);
        } else if (pos >= sh && (pos - sh) % S == 0) {
          const int j = (pos - sh) / S;
          if (j < NRH && early_slot(h, j)) issue_tok_node(h, j, node);
        }
      }
      base += __popc(wv);
    }
    if (nxt >= 1 && lane == 0) {   // the orphans of the next level
      const int nch = p.b * kap, a0 = max(nch, lo2), a1 = min(cnt_c[nxt], hi2);
      if (a1 > a0)
        bulk_g2s(kdst + size_t(a0 - lo2) * D,
                 ksrc + (int64_t(p.b) * vis[lev] + (a0 - nch)) * D, unsigned(a1 - a0) * rb,
                 mb_lev);
    }
    __syncwarp();
    if (lane == 0)   // the producer reads the kept list (one arrival per head)
      for (int n = 0; n < (grp ? HPC : 1); ++n) mbar_arrive(mb_kept);
  };

  // Level barrier: the head group's scores of this level are complete and
  // visible in this CTA.  With S > 1 every CTA of the group arrives on the
  // group's "ready" barrier of the level's parity: a CTA can be at most one
  // level ahead of another (it waits for everyone's arrival), so alternating
  // two barriers keeps the arrivals of consecutive levels apart.
  int use = 0;   // levels passed (mb_lev phase; mb_ready[use & 1] phase use / 2)
  auto level_sync = [&]() {
    if (S == 1) {
      named_sync(kBarChain, kChainThreads);
    } else {
      fence_cluster();
      named_sync(kBarChain, kChainThreads);
      uint64_t* rb = mb_ready + (use & 1);
      if (tid < S) mbar_arrive_remote(rb, hg * S + tid);
      mbar_wait(rb, unsigned(use >> 1) & 1u, timed_out);
    }
  };

  // Kept-leaf tokens of head hw through its ring of NRH slots, two rows per
  // slot at a time.  Leaf j of the share has rank sh + j * S, so its row e
  // sits at RoPE index (sh + j S) B + e; as for the summaries, the query
  // (rotated to n0 - 1 in qtok) is turned back by each row's index: the seed
  // R((sh + j S) B) advances by R(S B) per leaf and is combined with the
  // slot's R(hs), and the query turns by R(-HSLOT) per row.
  auto token_pass = [&]() {
    float qt[8];
    lds_pairs(qtok + (hg * HPC + hw) * D, j0, HALF, qt);
    const unsigned lbar = kBarHead0 + hw;
    float rj[8], st2[8];
    if (p.rope) {
      lds_cs8(rrow + p.lay.levels * D, j0, rj);
      cmul8(st2, cs_st, cs_st);
    }
    const size_t slot_elems = size_t(2) * p.B * D;
    // With S = 1 two consecutive leaves of the share sit at consecutive RoPE
    // indices, so they are processed as one block of 2B rows (fewer, fuller
    // iterations and one barrier per pair).
    for (int j = 0; j < ntok;) {
      const int nl = (S == 1 && NRH >= 2 && j + 1 < ntok) ? 2 : 1;
      const int slot0 = j % NRH, slot1 = (j + 1) % NRH;
      mbar_wait(mb_tok + hb * NRH + slot0, unsigned(j / NRH) & 1u, timed_out);
      if (nl == 2) mbar_wait(mb_tok + hb * NRH + slot1, unsigned((j + 1) / NRH) & 1u, timed_out);
      const T* cK0 = tbuf + (size_t(hb) * NRH + slot0) * slot_elems;
      const T* cK1 = tbuf + (size_t(hb) * NRH + slot1) * slot_elems;
      float q0[8];
      if (p.rope) {
        float seed[8], r[8], t2[8];
        cmul8(seed, rj, cs_hs);
        rot_neg8(q0, qt, seed);
        lds_cs8(rrow + (p.lay.levels + 1) * D, j0, r);
        for (int x = 0; x < nl; ++x) {
          cmul8(t2, rj, r);
#pragma unroll
          for (int c = 0; c < 8; ++c) rj[c] = t2[c];
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) q0[c] = qt[c];
      }
      const int nrow = nl * p.B;
      for (int e = hs; e - hs < nrow; e += 2 * HSLOT) {
        const int e1 = e + HSLOT;
        const bool on0 = e < nrow, on1 = e1 < nrow;
        const int r0 = on0 ? e : 0, r1 = on1 ? e1 : 0;
        const T* k0p = (r0 < p.B ? cK0 + size_t(r0) * D : cK1 + size_t(r0 - p.B) * D);
        const T* k1p = (r1 < p.B ? cK0 + size_t(r1) * D : cK1 + size_t(r1 - p.B) * D);
        float k0[8], k1[8], v0[8], v1[8], q1[8];
        SharedPairs<T, HALF>::load(k0p, j0, k0);
        SharedPairs<T, HALF>::load(k1p, j0, k1);
        SharedPairs<T, HALF>::load(k0p + size_t(p.B) * D, j0, v0);
        SharedPairs<T, HALF>::load(k1p + size_t(p.B) * D, j0, v1);
        if (p.rope) {
          rot_neg8(q1, q0, cs_st);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) q1[c] = q0[c];
        }
        float s0 = dot8(q0, k0), s1 = dot8(q1, k1);
        if (p.rope) {
          float t[8];
          rot_neg8(t, q0, st2);
#pragma unroll
          for (int c = 0; c < 8; ++c) q0[c] = t[c];
        }
        slot_sum2<LPR>(s0, s1);
        fold2(m, l, acc, s0 * inv_sqrt_d, on0, v0, s1 * inv_sqrt_d, on1, v1);
      }
      named_sync(lbar, WPH * 32);
      if (warp == hw * WPH && lane == 0) {
        if (j + NRH < ntok) mbar_arrive(mb_empty + hb * NRH + slot0);
        if (nl == 2 && j + 1 + NRH < ntok) mbar_arrive(mb_empty + hb * NRH + slot1);
      }
      j += nl;
    }
  };

  auto chain_warps = [&]() {
    for (int lev = top; lev >= 1; --lev) {
      mbar_wait(mb_lev, unsigned(use) & 1u, timed_out);
      score_level(lev);
      level_sync();
      const int u = use++;
      if (grp && cnt_k[lev] < cnt_c[lev]) group_scores(lev);
      if (warp >= 4 - HPC && warp < 4) select_level(lev);
      named_sync(kBarChain, kChainThreads);
      mbar_wait(mb_val, unsigned(u) & 1u, timed_out);
      fold_values(lev);
      named_sync(kBarChain, kChainThreads);
      if (tid == 0) mbar_arrive(mb_folded);
    }
    if (top > 0) token_pass();
    // Expiry test: with the work done, one more bounded wait on a barrier that
    // no thread arrives at; it runs out and the launch reports the timeout.
    if (p.test_expire) mbar_wait(mb_never, 0u, timed_out);
  };

  // The producer warp issues the chain's other copies: a level's values once
  // the level above is folded (vbuf is free) and the level's keys have landed,
  // the kept leaves of level 1 whose ring slots reach into vbuf (once it is
  // free), and each ring slot again when its head's warps have consumed it.
  // (The top level's copies are issued before the query is loaded; the keys
  // of the levels below and the kept leaves in kbuf by the selection warps.)
  auto producer_warp = [&]() {
    for (int u = 0; u < top; ++u) {
      const int lev = top - u;
      mbar_wait(mb_kept, unsigned(u) & 1u, timed_out);
      mbar_wait(mb_folded, unsigned(u) & 1u, timed_out);
      // the next level's values are not needed before its top-k: let its keys
      // land first, so that they get the memory bandwidth to themselves
      if (lev > 1) mbar_wait(mb_lev, unsigned(u + 1) & 1u, timed_out);
      if (lane == 0) fence_proxy_async();
      __syncwarp();
      if (lev > 1) {
        issue_level(lev - 1, true);
      } else if (lane < HB) {
        for (int j = 0; j < NRH && j < ntok; ++j)
          if (!early_slot(lane, j)) issue_tok(lane, j);
      }
    }
    if (top > 0 && lane < HB) {
      const int h = lane;
      for (int j = NRH; j < ntok; ++j) {
        mbar_wait(mb_empty + h * NRH + j % NRH, unsigned(j / NRH - 1) & 1u, timed_out);
        fence_proxy_async();
        issue_tok(h, j);
      }
    }
  };

  if (warp == kProducerWarp)
    producer_warp();
  else if (warp >= kChainWarps)
    window_warps();
  else
    chain_warps();

  // ---- merge ----------------------------------------------------------------
  // The slots of a chain warp, then per head the head's chain warps plus the
  // window partials; each CTA sends its contribution for every head of the
  // group to the head's owner (share 0 of its head group), which combines the
  // CS contributions and writes O.
  if (warp < kChainWarps) {
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) merge_xor(m, l, acc, o);
    if (lane < LPR) {
      float* w = wsc + warp * RS;
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
  }
  if (timed_out) {
    // the launch's output is not valid; give copies still in flight into this
    // CTA's shared memory time to land before the CTA can exit
    atomicOr(errw, RECSA_DEVERR_WAIT_TIMEOUT);
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 1000000ull) __nanosleep(10000);
  }
  __syncthreads();
  for (int x = tid; x < G * D; x += kThreads) {
    const int h = x / D, c = x % D;
    const int lh = h % HPC;
    const bool mine = h / HPC == hg;
    float mm = -INFINITY;
    if (mine)
      for (int w = lh * WPH; w < (lh + 1) * WPH; ++w) mm = fmaxf(mm, wsc[w * RS + D]);
    for (int w = 0; w < kWinWarps; ++w) mm = fmaxf(mm, wwin[(w * G + h) * RS + D]);
    float aa = 0.f, ll = 0.f;
    if (mm != -INFINITY) {
      if (mine)
        for (int w = lh * WPH; w < (lh + 1) * WPH; ++w) {
          const float* ws = wsc + w * RS;
          const float r = (ws[D] == -INFINITY) ? 0.f : __expf(ws[D] - mm);
          aa = fmaf(ws[c], r, aa);
          ll = fmaf(ws[D + 1], r, ll);
        }
      for (int w = 0; w < kWinWarps; ++w) {
        const float* ws = wwin + (w * G + h) * RS;
        const float r = (ws[D] == -INFINITY) ? 0.f : __expf(ws[D] - mm);
        aa = fmaf(ws[c], r, aa);
        ll = fmaf(ws[D + 1], r, ll);
      }
    }
    float* dst = (CS == 1 ? mrg : cluster.map_shared_rank(mrg, (h / HPC) * S)) +
                 (rank * HPC + lh) * RS;
    dst[c] = aa;
    if (c == 0) {
      dst[D] = mm;
      dst[D + 1] = ll;
    }
  }
  if (CS > 1)
    cluster.sync();
  else
    __syncthreads();
  if (sh == 0) {
    for (int x = tid; x < HPC * D; x += kThreads) {
      const int h = x / D, c = x % D;
      float mm = -INFINITY;
      for (int r = 0; r < CS; ++r) mm = fmaxf(mm, mrg[(r * HPC + h) * RS + D]);
      float aa = 0.f, ll = 0.f;
      if (mm != -INFINITY)
        for (int r = 0; r < CS; ++r) {
          const float* ms = mrg + (r * HPC + h) * RS;
          const float w = (ms[D] == -INFINITY) ? 0.f : __expf(ms[D] - mm);
          aa = fmaf(ms[c], w, aa);
          ll = fmaf(ms[D + 1], w, ll);
        }
      const float o = (empty || ll == 0.f) ? 0.f : aa / ll;
      store_elem(O, qrow + int64_t(hg * HPC + h) * D + c, o, p.dtype);
    }
    if (trace && !empty) {
      for (int x = tid; x < HPC * kTraceHead; x += kThreads) {
        const int h = x / kTraceHead, f = x % kTraceHead;
        const int64_t rec =
            ((seq * n_q + qi) * p.hq + int64_t(g) * G + hg * HPC + h) * tstride;
        int v = 0;
        if (f == 0) v = top;
        else if (f == 1 || f == 2 || f == 3) {
          int64_t e = 0, r = 0;
          for (int lev = 1; lev <= top; ++lev) { e += cnt_c[lev] - cnt_k[lev]; r += cnt_c[lev]; }
          v = int(f == 1 ? e + n0 : f == 2 ? r + n0 : n0);
        } else if (f < 4 + kMaxLevels) {
          const int lev = f - 4 + 1;
          v = lev <= top ? cnt_c[lev] : 0;
        } else {
          const int lev = f - 4 - kMaxLevels + 1;
          v = lev <= top ? cnt_k[lev] : 0;
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
      if ((t + 1) % p.B == 0 && warp == 0)
        pool_appended<T, D>(p, K, V, tree, st.r + g * st.r_stride, kvbase, t, seq, g, lane);
    }
    // Length: every cluster of the sequence read len at its start; the last
    // one to finish (per-sequence counter) publishes len + 1 and resets it.
    if (rank == 0 && tid == 0) {
      if (!do_append) {
        if (len0 >= p.cap) atomicOr(errw, RECSA_DEVERR_APPEND_FULL);
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

template <typename T, int D, int G, int HPC>
cudaError_t cluster_typed(const Params& p, const void* Q, const void* K, const void* V,
                          const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                          int32_t* trace, cudaStream_t s, int S, StepArgs st) {
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  int64_t cm = p.b * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  const int cmax = int(cm < 1 ? 1 : cm);
  const int kmax = int(kk < cmax ? kk : cmax);
  if (cmax > 32 * kRegSlots * 4) return cudaErrorNotSupported;
  // The most kept-leaf ring slots that fit; more shares per head group when
  // even one slot (or one share of a level's keys) does not fit.
  int cs = (G / HPC) * S, nrh = 0;
  Plan pl{};
  for (;;) {
    if (cs > kMaxCluster) return cudaErrorNotSupported;
    for (nrh = kMaxTokSlots; nrh >= 1; --nrh) {
      pl = make_plan<T, D, G, HPC>(cmax, kmax, S, cs, nrh, p.B, p.lay.levels,
                                   p.mode == RECSA_MODE_GROUP ? 1 : HPC);
      if (pl.total <= kSmemLimit) break;
    }
    if (nrh >= 1) break;
    S *= 2;
    cs *= 2;
  }
  auto kern = decode_cluster_kernel<T, D, G, HPC>;
  cudaError_t e = ensure_smem(kern, int(pl.total));
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = ensure_nonportable_cluster(kern);
    if (e != cudaSuccess) return e;
  }
  if (int64_t(p.batch) * p.hkv > 65535 || n_q > 65535) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, n_q, unsigned(p.batch * p.hkv));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.total;
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
                            len_dev, int(n_q), reinterpret_cast<T*>(O), trace, cmax, kmax, S,
                            nrh, st);
}

template <typename T, int D>
cudaError_t cluster_g(const Params& p, const void* Q, const void* K, const void* V,
                      const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                      int32_t* trace, cudaStream_t s, int hpc, int S, StepArgs st) {
#define RECSA_CLUSTER_CASE(GG, HH)                                                          \
  if (p.group == GG && hpc == HH)                                                           \
    return cluster_typed<T, D, GG, HH>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, S, st);
  RECSA_CLUSTER_CASE(1, 1)
  RECSA_CLUSTER_CASE(2, 1)
  RECSA_CLUSTER_CASE(2, 2)
  RECSA_CLUSTER_CASE(4, 1)
  RECSA_CLUSTER_CASE(4, 2)
  RECSA_CLUSTER_CASE(4, 4)
#undef RECSA_CLUSTER_CASE
  return cudaErrorNotSupported;
}

// Heads per CTA (HPC) and candidate shares per head group (S) of a launch.
// RECSA_DECODE_SPLIT="hpc,s" forces both (tests); otherwise the rule below.
// (The launch doubles S further when a share's rows do not fit shared memory.)
void decode_split(const Params& p, int32_t n_q, int& hpc, int& S) {
  const int G = p.group;
  const Switches& sw = switches();
  if (sw.split_hpc) {
    const int h = sw.split_hpc, s = sw.split_s;
    if (h <= G && G % h == 0 && (h & (h - 1)) == 0 && (s & (s - 1)) == 0 &&
        (G / h) * s <= kMaxCluster) {
      hpc = h;
      S = s;
      return;
    }
  }
  const int64_t pairs = int64_t(p.batch) * p.hkv * n_q;
  if (p.mode == RECSA_MODE_GROUP) {
    // every head of the group in one CTA; shares fill the 148 SMs
    hpc = G;
    S = 1;
    while (S * 2 <= kMaxCluster && pairs * S * 2 <= 148) S *= 2;
    return;
  }
  // One query head per CTA, and a second candidate share when the grid still
  // fits the 148 SMs.  Measured at 131K and 2M (batch 1), 1M (batch 8) and
  // 524K (batch 4): more heads per CTA or more shares cost more in per-CTA
  // work and cross-CTA level barriers than the extra SMs give back, even when
  // the grid then needs several waves.
  hpc = 1;
  S = pairs * G * 2 <= 148 ? 2 : 1;
}

cudaError_t cluster_dispatch(const Params& p, const void* Q, const void* K, const void* V,
                             const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                             int32_t* trace, cudaStream_t s, StepArgs st) {
  int hpc = 1, S = 1;
  decode_split(p, n_q, hpc, S);
  // group selection needs every head's scores in each CTA
  if (p.mode == RECSA_MODE_GROUP && hpc != p.group) return cudaErrorNotSupported;
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128
               ? cluster_g<__nv_bfloat16, 128>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, hpc, S, st)
               : cluster_g<__nv_bfloat16, 64>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, hpc, S, st);
  return p.d == 128 ? cluster_g<float, 128>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, hpc, S, st)
                    : cluster_g<float, 64>(p, Q, K, V, tree, len_dev, n_q, O, trace, s, hpc, S, st);
}

}  // namespace

cudaError_t launch_decode_cluster(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, const int64_t* len_dev, int32_t n_q, void* O,
                                  int32_t* trace, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA && p.mode != RECSA_MODE_GROUP) return cudaErrorNotSupported;
  StepArgs st = {};
  return cluster_dispatch(p, Q, K, V, tree, len_dev, n_q, O, trace, s, st);
}

cudaError_t launch_decode_step(const Params& p, const void* Q, void* K, void* V,
                               const void* k_new, const void* v_new, int64_t* len_dev,
                               const float* r, int64_t r_stride, void* tree, int32_t n_q,
                               void* O, int32_t* trace, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA && p.mode != RECSA_MODE_GROUP) return cudaErrorNotSupported;
  if (p.batch > kStepCounters) return cudaErrorNotSupported;
  StepArgs st;
  st.k_new = k_new;
  st.v_new = v_new;
  st.r = r;
  st.r_stride = r_stride;
  st.len_w = len_dev;
  st.counters = reinterpret_cast<int*>(reinterpret_cast<char*>(tree) + kStepCounterOffset);
  st.fuse = 1;
  return cluster_dispatch(p, Q, K, V, tree, len_dev, n_q, O, trace, s, st);
}

}  // namespace recsa
