// ZHA routing variant ("Subquadratic Attention with a Hierarchical
// Tree-Structured Indexer", Figure 3 caption): one CTA per (query, sequence,
// query head).
//
// Per query at position t:
//   * routing, top-down over the visible levels: candidates = children of the
//     nodes expanded one level up, then the orphans; score = q . key / sqrt(d)
//     on the un-rotated query and summary key; the expanded set is the
//     shortest prefix in decreasing-score order (ties -> lower index) whose
//     softmax mass over the level's candidates reaches top_p, capped at
//     min(k, c); no summary enters the attention;
//   * attention: one softmax over the tokens of the reached leaves and the
//     exact window [a*B, t], at their true positions with standard RoPE.
//
// Layout for B200:
//   * Warps 0-11 (the chain) walk the levels: a level's candidate key rows are
//     copied into shared memory with 16-byte cp.async (the whole level in
//     flight at once) and scored four rows per warp at a time; the top-p cut
//     comes from every candidate's rank (one chain thread per candidate) and
//     a warp scan of the weights laid out by rank.
//   * Warps 12-15 attend the window, which does not depend on the routing,
//     while the chain runs; then all 16 warps attend the reached leaves.
//   * Exact tokens are taken in units of up to 16 consecutive positions: the
//     query is rotated once per unit by R(t - first position) from the RoPE
//     table and turned by R(-1) per following token, so a key is never
//     rotated.  A warp loads a whole unit's K and V rows (bf16; half a unit
//     for fp32) into registers, still packed, before it uses any of them.
//   * Each warp keeps an online softmax (max, sum, its lanes' channels of the
//     accumulator); the 16 states are merged through shared memory.
#include <algorithm>

#include "recsa_internal.cuh"

namespace recsa {
namespace {

// Launch shapes: decode (and prefill without window partials) runs 12 routing
// warps and 4 window warps per query head; prefill with the tensor-core
// window kernel's partials runs 4 routing warps and no window warps, in a
// CTA small enough for four to share an SM.
constexpr int kZDecChain = 12, kZDecWin = 4;
constexpr int kZPreChain = 4;
constexpr int kZMaxCand = 1024;     // candidates per level (smem per CTA)
constexpr size_t kZStageBytes = 180 * 1024;   // shared memory for a level's staged key rows
constexpr int kZUnit = 16;          // consecutive exact tokens per work unit
constexpr int kZBarChain = 1;       // named barrier of the chain warps

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
// 4- and 8-byte copies (row scales, NVFP4 block scales), also asynchronous.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}
template <int NTH>
__device__ __forceinline__ void chain_sync() {
  asm volatile("bar.sync %0, %1;\n" ::"n"(kZBarChain), "n"(NTH) : "memory");
}

// Lane l holds channel pairs (NP * l + u, NP * l + u + D/2), u < NP, of a row.
template <int NP>
__device__ __forceinline__ void load_pairs(const float* row, int lane, float (&x1)[NP],
                                           float (&x2)[NP]) {
  constexpr int HALF = 32 * NP;
  if constexpr (NP == 2) {
    const float2 a = *reinterpret_cast<const float2*>(row + 2 * lane);
    const float2 b = *reinterpret_cast<const float2*>(row + HALF + 2 * lane);
    x1[0] = a.x; x1[1] = a.y; x2[0] = b.x; x2[1] = b.y;
  } else {
    x1[0] = row[lane];
    x2[0] = row[HALF + lane];
  }
}
template <int NP>
__device__ __forceinline__ void load_pairs(const __nv_bfloat16* row, int lane, float (&x1)[NP],
                                           float (&x2)[NP]) {
  constexpr int HALF = 32 * NP;
  if constexpr (NP == 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + 2 * lane));
    const float2 b =
        __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + HALF + 2 * lane));
    x1[0] = a.x; x1[1] = a.y; x2[0] = b.x; x2[1] = b.y;
  } else {
    x1[0] = __bfloat162float(row[lane]);
    x2[0] = __bfloat162float(row[HALF + lane]);
  }
}

// The lane's slice of a row as loaded (not yet converted): pairs
// (NP * l + u) and (NP * l + u + D/2).
template <typename T, int NP> struct Raw;
template <> struct Raw<__nv_bfloat16, 2> { __nv_bfloat162 a, b; };
template <> struct Raw<__nv_bfloat16, 1> { __nv_bfloat16 a, b; };
template <> struct Raw<float, 2> { float2 a, b; };
template <> struct Raw<float, 1> { float a, b; };

// The lane's channels of an FP8 code row (decoded, before the row's scale).
template <int NP>
__device__ __forceinline__ void load_codes(const unsigned char* row, int lane, float (&x1)[NP],
                                           float (&x2)[NP]) {
  constexpr int HALF = 32 * NP;
  if constexpr (NP == 2) {
    const unsigned short a = *reinterpret_cast<const unsigned short*>(row + 2 * lane);
    const unsigned short b = *reinterpret_cast<const unsigned short*>(row + HALF + 2 * lane);
    x1[0] = fp8_to_float(a & 0xFF); x1[1] = fp8_to_float(a >> 8);
    x2[0] = fp8_to_float(b & 0xFF); x2[1] = fp8_to_float(b >> 8);
  } else {
    x1[0] = fp8_to_float(row[lane]);
    x2[0] = fp8_to_float(row[HALF + lane]);
  }
}

// The lane's channels of an NVFP4 code row: E2M1 values times their block's
// E4M3 scale (before the row's scale).  Element e is nibble e & 1 of byte e / 2
// and belongs to block e / 16.
template <int NP>
__device__ __forceinline__ void load_codes_nvfp4(const unsigned char* row,
                                                 const unsigned char* bsc, int lane,
                                                 float (&x1)[NP], float (&x2)[NP]) {
  constexpr int HALF = 32 * NP;
  if constexpr (NP == 2) {   // elements 2l, 2l + 1 and HALF + 2l, HALF + 2l + 1
    const unsigned a = row[lane], b = row[HALF / 2 + lane];
    const float sa = fp8_to_float(bsc[lane >> 3]), sb = fp8_to_float(bsc[(HALF >> 4) + (lane >> 3)]);
    x1[0] = fp4_to_float(a) * sa; x1[1] = fp4_to_float(a >> 4) * sa;
    x2[0] = fp4_to_float(b) * sb; x2[1] = fp4_to_float(b >> 4) * sb;
  } else {                   // elements l and HALF + l
    const int sh = 4 * (lane & 1);
    x1[0] = fp4_to_float(row[lane >> 1] >> sh) * fp8_to_float(bsc[lane >> 4]);
    x2[0] = fp4_to_float(row[(HALF + lane) >> 1] >> sh) * fp8_to_float(bsc[(HALF + lane) >> 4]);
  }
}

template <typename T, int NP>
__device__ __forceinline__ Raw<T, NP> load_raw(const T* row, int lane) {
  constexpr int HALF = 32 * NP;
  Raw<T, NP> r;
  if constexpr (NP == 2) {
    using P2 = decltype(r.a);
    r.a = *reinterpret_cast<const P2*>(row + 2 * lane);
    r.b = *reinterpret_cast<const P2*>(row + HALF + 2 * lane);
  } else {
    r.a = row[lane];
    r.b = row[HALF + lane];
  }
  return r;
}
template <typename T, int NP>
__device__ __forceinline__ void unpack(const Raw<T, NP>& r, float (&x1)[NP], float (&x2)[NP]) {
  if constexpr (NP == 2) {
    if constexpr (sizeof(T) == 2) {
      const float2 a = __bfloat1622float2(r.a), b = __bfloat1622float2(r.b);
      x1[0] = a.x; x1[1] = a.y; x2[0] = b.x; x2[1] = b.y;
    } else {
      x1[0] = r.a.x; x1[1] = r.a.y; x2[0] = r.b.x; x2[1] = r.b.y;
    }
  } else {
    if constexpr (sizeof(T) == 2) {
      x1[0] = __bfloat162float(r.a);
      x2[0] = __bfloat162float(r.b);
    } else {
      x1[0] = r.a;
      x2[0] = r.b;
    }
  }
}

// NCH routing-chain warps, NWIN window warps; NWIN = 0 takes the window's
// softmax state from wpart (the window kernel's partials, per query head:
// normalised output [D], max, sum).
template <typename T, int NP, int NCH, int NWIN>
__global__ void __launch_bounds__((NCH + NWIN) * 32, NWIN == 0 ? 4 : 1)
zha_attend_kernel(Params p, const T* __restrict__ Q, const T* __restrict__ K,
                  const T* __restrict__ V, const void* __restrict__ tree,
                  const int64_t* __restrict__ len_dev, int64_t q_start, int n_q, int decode,
                  T* __restrict__ O, int32_t* __restrict__ trace, int cmax, int kmax,
                  int krows, const float* __restrict__ wpart) {
  constexpr int D = 64 * NP, HALF = 32 * NP;
  constexpr int NW = NCH + NWIN, NT = NW * 32, CT = NCH * 32;
  constexpr int RS = D + 2;                      // warp state row: acc[D], m, l
  const int qi = blockIdx.x;
  const int64_t seq = blockIdx.y;
  const int h = blockIdx.z;                      // query head
  const int g = h / p.group;                     // its KV head
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smem[];
  const bool fp8 = p.kfmt == RECSA_KEYS_FP8;                  // FP8 key codes + row scales
  const bool nv4 = p.kfmt == RECSA_KEYS_NVFP4;                // E2M1 codes + block, row scales
  const bool lowp = fp8 || nv4;
  const int rowb = fp8 ? D : (nv4 ? D / 2 + D / 16 : 4 * D);  // staged bytes per key row
  float* kbuf = reinterpret_cast<float*>(smem);               // [krows][D] level key rows
  const unsigned char* kbyte = smem;                          // (FP8: [krows][D] codes;
  unsigned char* kbs = smem + size_t(krows) * (D / 2);        //  NVFP4: [krows][D/2] codes,
                                                              //  then [krows][D/16] scales)
  float* rowsc = reinterpret_cast<float*>(smem + size_t(krows) * rowb);
  float* ksc = rowsc + krows;                                 // [krows] FP8 row scales
  float* score = ksc + krows;                                 // [cmax]
  float* wsort = score + cmax;                                // [cmax] weights by rank
  float* zsum = wsort + cmax;                                 // [NCH] sums, [NCH] max
  float* wst = zsum + NCH + 1;                                // [NW][RS] warp states
  int* kept = reinterpret_cast<int*>(wst + NW * RS);          // [2][kmax] by level parity
  int* zc = kept + 2 * kmax;                                  // [kMaxLevels + 1] candidates
  int* zk = zc + kMaxLevels + 1;                              // [kMaxLevels + 1] expanded
  int* rankv = zk + kMaxLevels + 1;                           // [cmax] candidate ranks
  int* zcnt = rankv + cmax;                                   // [rounds][NCH] expanded

  const int64_t t = decode ? len_dev[seq] - 1 : q_start + qi;
  const int64_t orow = ((seq * n_q + qi) * p.hq + h) * D;
  if (t < 0 || t >= p.cap) {   // empty sequence, or a length beyond capacity: zeros
    for (int x = tid; x < D; x += NT) O[orow + x] = T(0.f);
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
  const int64_t kvbase = (seq * p.hkv + g) * p.cap;
  const int64_t n_win = t + 1 - a * p.B;
  const int tstride = kTraceHead + kMaxLevels * p.k;
  int32_t* rec = trace ? trace + ((seq * n_q + qi) * p.hq + h) * tstride : nullptr;

  // The lane's channels of the raw query, and R(-1) for the per-token turn.
  float q1[NP], q2[NP], c1[NP], s1[NP];
  load_pairs<NP>(Q + orow, lane, q1, q2);
#pragma unroll
  for (int u = 0; u < NP; ++u) {
    c1[u] = 1.f;
    s1[u] = 0.f;
    if (p.rope) {
      const float2 cs = rope[HALF + NP * lane + u];    // table row 1
      c1[u] = cs.x;
      s1[u] = cs.y;
    }
  }

  // Online softmax of this warp: m, l (warp-uniform) and the lane's channels.
  float m_run = -INFINITY, l_run = 0.f, acc1[NP], acc2[NP];
#pragma unroll
  for (int u = 0; u < NP; ++u) acc1[u] = acc2[u] = 0.f;

  // Exact tokens [pos0, pos0 + n), n <= kZUnit, at their true positions.
  auto attend_unit = [&](int64_t pos0, int n) {
    float r1[NP], r2[NP];   // query rotated by R(t - pos) for the current token
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      r1[u] = q1[u];
      r2[u] = q2[u];
      if (p.rope) {
        const float2 cs = rope[(t - pos0) * HALF + NP * lane + u];
        r1[u] = q1[u] * cs.x - q2[u] * cs.y;
        r2[u] = q2[u] * cs.x + q1[u] * cs.y;
      }
    }
    constexpr int TB = sizeof(T) == 2 ? kZUnit : kZUnit / 2;   // tokens per batch
    for (int b0 = 0; b0 < n; b0 += TB) {
      const int nb = n - b0 < TB ? n - b0 : TB;
      Raw<T, NP> kr[TB], vr[TB];
#pragma unroll
      for (int i = 0; i < TB; ++i) {   // every load first (rows past nb repeat the last)
        const int64_t row = (kvbase + pos0 + b0 + (i < nb ? i : nb - 1)) * D;
        kr[i] = load_raw<T, NP>(K + row, lane);
        vr[i] = load_raw<T, NP>(V + row, lane);
      }
      float s[TB];
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        float k1[NP], k2[NP];
        unpack<T, NP>(kr[i], k1, k2);
        float d_ = 0.f;
#pragma unroll
        for (int u = 0; u < NP; ++u) {
          d_ = fmaf(r1[u], k1[u], d_);
          d_ = fmaf(r2[u], k2[u], d_);
          // turn the query by R(-1): the next token is one position later
          const float x1 = r1[u], x2 = r2[u];
          r1[u] = x1 * c1[u] + x2 * s1[u];
          r2[u] = x2 * c1[u] - x1 * s1[u];
        }
        s[i] = d_;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int i = 0; i < TB; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
      float mx = m_run;
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        s[i] = i < nb ? s[i] * p.inv_sqrt_d : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float scale = expf(m_run - mx);
      l_run *= scale;
#pragma unroll
      for (int u = 0; u < NP; ++u) {
        acc1[u] *= scale;
        acc2[u] *= scale;
      }
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        const float w = expf(s[i] - mx);   // 0 past nb
        float v1[NP], v2[NP];
        unpack<T, NP>(vr[i], v1, v2);
        l_run += w;
#pragma unroll
        for (int u = 0; u < NP; ++u) {
          acc1[u] = fmaf(w, v1[u], acc1[u]);
          acc2[u] = fmaf(w, v2[u], acc2[u]);
        }
      }
      m_run = mx;
    }
  };

  if (warp < NCH) {
    // ---- routing chain ----------------------------------------------------
    const int ct = tid;                          // 0 .. 255
    int kup = 0;
    for (int lev = top; lev >= 1; --lev) {
      const int64_t vup = lev < top ? vis[lev + 1] : 0;
      const int nch = p.b * kup;
      const int c = nch + int(vis[lev] - p.b * vup);
      const int* kprev = kept + ((lev + 1) & 1) * kmax;
      auto node = [&](int i) -> int {
        return i < nch ? kprev[div_b(p, i)] * p.b + mod_b(p, i) : int(p.b * vup) + (i - nch);
      };
      const float* keys = level_keys(p, const_cast<void*>(tree), lev, seq, g);
      // A node holds R = nref keys (one per reference query) and scores its
      // best match.  The level's rows (candidate, reference) go through kbuf
      // in chunks of krows / R candidates; with R = 1 that is one chunk.
      const int R = p.nref;
      const int cc = krows / R;
      const unsigned char* kcodes = level_kcodes(p, const_cast<void*>(tree), lev, seq, g);
      const float* kscales = level_kscales(p, const_cast<void*>(tree), lev, seq, g);
      const unsigned char* kbsc = level_kbscales(p, const_cast<void*>(tree), lev, seq, g);
      const int C16 = fp8 ? D / 16 : (nv4 ? D / 32 : D / 4);   // 16-byte pieces per row
      for (int i0c = 0; i0c < c; i0c += cc) {
        const int i1c = min(c, i0c + cc);
        const int nrow = (i1c - i0c) * R;
        for (int x = ct; x < nrow * C16; x += CT) {
          const int q = x / C16, pc = x % C16;
          const int i = i0c + q / R, ref = q % R;
          const int64_t row = int64_t(node(i)) * R + ref;
          if (fp8)
            cp_async16(const_cast<unsigned char*>(kbyte) + size_t(q) * D + pc * 16,
                       kcodes + row * D + pc * 16);
          else if (nv4)
            cp_async16(const_cast<unsigned char*>(kbyte) + size_t(q) * (D / 2) + pc * 16,
                       kcodes + row * (D / 2) + pc * 16);
          else
            cp_async16(kbuf + size_t(q) * D + pc * 4, keys + row * D + pc * 4);
        }
        if (lowp)   // row scales (and NVFP4 block scales) ride with the code rows
          for (int q = ct; q < nrow; q += CT) {
            const int64_t row = int64_t(node(i0c + q / R)) * R + q % R;
            cp_async4(ksc + q, kscales + row);
            if (nv4) {   // D / 16 block-scale bytes (8 at D = 128, 4 at D = 64)
              if constexpr (D == 128)
                cp_async8(kbs + size_t(q) * 8, kbsc + row * 8);
              else
                cp_async4(kbs + size_t(q) * 4, kbsc + row * 4);
            }
          }
        cp_async_wait_all();
        chain_sync<CT>();
        float* rsc = R == 1 ? score + i0c : rowsc;   // row scores
        // rows warp, warp + 8, ...; four rows per warp at a time
        for (int q0 = warp; q0 < nrow; q0 += 4 * NCH) {
          float sc4[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int q = min(q0 + r * NCH, nrow - 1);   // rows past nrow repeat the last
            float x1[NP], x2[NP];
            if (fp8)
              load_codes<NP>(kbyte + size_t(q) * D, lane, x1, x2);
            else if (nv4)
              load_codes_nvfp4<NP>(kbyte + size_t(q) * (D / 2), kbs + size_t(q) * (D / 16), lane,
                                   x1, x2);
            else
              load_pairs<NP>(kbuf + size_t(q) * D, lane, x1, x2);
            sc4[r] = 0.f;
#pragma unroll
            for (int u = 0; u < NP; ++u) {
              sc4[r] = fmaf(q1[u], x1[u], sc4[r]);
              sc4[r] = fmaf(q2[u], x2[u], sc4[r]);
            }
          }
          // the four rows' sums by a transposed reduction (6 shuffles, not 20):
          // across lanes 16 apart each lane keeps two of the rows, across
          // lanes 8 apart one, then the remaining lanes fold; lane 8 r (r < 4)
          // ends with row r's sum
          const bool u4 = (lane >> 4) & 1, u3 = (lane >> 3) & 1;
          float a0 = u4 ? sc4[2] : sc4[0], a1 = u4 ? sc4[3] : sc4[1];
          a0 += __shfl_xor_sync(0xffffffffu, u4 ? sc4[0] : sc4[2], 16);
          a1 += __shfl_xor_sync(0xffffffffu, u4 ? sc4[1] : sc4[3], 16);
          float v = u3 ? a1 : a0;
          v += __shfl_xor_sync(0xffffffffu, u3 ? a0 : a1, 8);
#pragma unroll
          for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if ((lane & 7) == 0) {
            const int q = q0 + (lane >> 3) * NCH;
            if (q < nrow) rsc[q] = v * p.inv_sqrt_d * (lowp ? ksc[q] : 1.f);
          }
        }
        chain_sync<CT>();
        if (R > 1) {   // a candidate's score: the best of its R rows
          for (int i = i0c + ct; i < i1c; i += CT) {
            float m = rsc[(i - i0c) * R];
            for (int ref = 1; ref < R; ++ref) m = fmaxf(m, rsc[(i - i0c) * R + ref]);
            score[i] = m;
          }
          chain_sync<CT>();
        }
      }
      chain_sync<CT>();
      // Top-p by ranks: chain thread ct holds candidates ct, ct + CT, ...  A
      // rank counts the better candidates (higher score, or equal at a lower
      // index); the weights exp(s - max) are laid out by rank, and warp 0
      // scans them for the shortest prefix whose mass reaches top_p of the
      // total, capped at min(k, c).
      for (int i = ct; i < c; i += CT) {
        const float si = score[i];
        int ri = 0;
        for (int j = 0; j < c; ++j) {
          const float sj = score[j];
          ri += (sj > si) || (sj == si && j < i);
        }
        rankv[i] = ri;
        if (ri == 0) zsum[NCH] = si;   // the level's maximum
      }
      chain_sync<CT>();
      float ws = 0.f;
      for (int i = ct; i < c; i += CT) {
        const float ei = expf(score[i] - zsum[NCH]);
        wsort[rankv[i]] = ei;
        ws += ei;
      }
      ws = warp_sum(ws);
      if (lane == 0) zsum[warp] = ws;
      chain_sync<CT>();
      if (warp == 0) {
        const float tot = warp_sum(lane < NCH ? zsum[lane] : 0.f);
        const float thr = p.top_p * tot;
        const int cap = c < p.k ? c : p.k;
        int cnt = cap;
        if (p.top_p < 1.f) {
          float run = 0.f;
          for (int b0 = 0; b0 < cap; b0 += 32) {
            const int e = b0 + lane;
            float x = e < cap ? wsort[e] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const float y = __shfl_up_sync(0xffffffffu, x, o);
              if (lane >= o) x += y;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, e < cap && run + x >= thr);
            if (hit) {
              cnt = b0 + __ffs(hit);
              break;
            }
            run += __shfl_sync(0xffffffffu, x, 31);
          }
        }
        if (lane == 0) {
          zc[lev] = c;
          zk[lev] = cnt;
        }
      }
      chain_sync<CT>();
      // expanded nodes in candidate order: rounds of CT candidates, a ballot
      // per warp and round, positions from the counts of earlier rounds/warps
      const int nrounds = (c + CT - 1) / CT;
      for (int r = 0; r < nrounds; ++r) {
        const int i = r * CT + ct;
        const unsigned bal = __ballot_sync(0xffffffffu, i < c && rankv[i] < zk[lev]);
        if (lane == 0) zcnt[r * NCH + warp] = __popc(bal);
      }
      chain_sync<CT>();
      int before = 0;
      for (int r = 0; r < nrounds; ++r) {
        const int i = r * CT + ct;
        const bool on = i < c && rankv[i] < zk[lev];
        const unsigned bal = __ballot_sync(0xffffffffu, on);
        if (on) {
          int pos = before + __popc(bal & ((1u << lane) - 1u));
          for (int w = 0; w < warp; ++w) pos += zcnt[r * NCH + w];
          const int id = node(i);
          kept[(lev & 1) * kmax + pos] = id;
          if (rec) rec[kTraceHead + (lev - 1) * p.k + pos] = id;
        }
        for (int w = 0; w < NCH; ++w) before += zcnt[r * NCH + w];
      }
      chain_sync<CT>();
      kup = zk[lev];
    }
  } else if constexpr (NWIN > 0) {
    // ---- window warps: [a*B, t], units of kZUnit positions ------------------
    const int nu = int((n_win + kZUnit - 1) / kZUnit);
    for (int u = warp - NCH; u < nu; u += NWIN) {
      const int64_t p0 = a * p.B + int64_t(u) * kZUnit;
      const int n = int(n_win - int64_t(u) * kZUnit < kZUnit ? n_win - int64_t(u) * kZUnit
                                                               : kZUnit);
      attend_unit(p0, n);
    }
  }
  __syncthreads();

  // ---- reached leaves: all warps ---------------------------------------------
  const int nleaf = top > 0 ? zk[1] : 0;
  const int upl = (p.B + kZUnit - 1) / kZUnit;   // units per leaf
  const int* leaves = kept + 1 * kmax;           // level 1 (odd parity)
  // the window warps take the first units: the chain warps start later
  for (int u = (warp + NW - NCH) % NW; u < nleaf * upl; u += NW) {
    const int r = u / upl, m = u % upl;
    const int n = p.B - m * kZUnit < kZUnit ? p.B - m * kZUnit : kZUnit;
    attend_unit(int64_t(leaves[r]) * p.B + m * kZUnit, n);
  }

  // ---- merge the warps' states ----------------------------------------------
  float* my = wst + warp * RS;
#pragma unroll
  for (int u = 0; u < NP; ++u) {
    my[NP * lane + u] = acc1[u];
    my[HALF + NP * lane + u] = acc2[u];
  }
  if (lane == 0) {
    my[D] = m_run;
    my[D + 1] = l_run;
  }
  __syncthreads();
  if (tid < D) {
    // the window's state: from the window warps, or the window kernel's partial
    const float* wrow = NWIN == 0 ? wpart + ((seq * n_q + qi) * p.hq + h) * (D + 2) : nullptr;
    float M = NWIN == 0 ? wrow[D] : -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wst[w * RS + D]);
    float L = 0.f, A = 0.f;
    if (NWIN == 0 && wrow[D] != -INFINITY) {
      const float e = expf(wrow[D] - M) * wrow[D + 1];   // normalised output x sum
      L = e;
      A = wrow[tid] * e;
    }
    for (int w = 0; w < NW; ++w) {
      const float mw = wst[w * RS + D];
      if (mw == -INFINITY) continue;
      const float e = expf(mw - M);
      L = fmaf(wst[w * RS + D + 1], e, L);
      A = fmaf(wst[w * RS + tid], e, A);
    }
    const float o = A / L;
    if constexpr (sizeof(T) == 2)
      O[orow + tid] = __float2bfloat16_rn(o);
    else
      O[orow + tid] = o;
  }
  if (rec && tid == 0) {
    const int64_t n0 = int64_t(nleaf) * p.B + n_win;
    int64_t keys_read = n0;
    for (int lev = 1; lev <= top; ++lev) keys_read += zc[lev];
    rec[0] = top;
    rec[1] = int32_t(n0);
    rec[2] = int32_t(keys_read);
    rec[3] = int32_t(n0);
    for (int lev = 1; lev <= kMaxLevels; ++lev) {
      const bool on = lev <= top;
      rec[4 + lev - 1] = on ? zc[lev] : 0;
      rec[4 + kMaxLevels + lev - 1] = on ? zk[lev] : 0;
    }
  }
}

template <typename T, int NP>
cudaError_t zha_typed(const Params& p, const void* Q, const void* K, const void* V,
                      const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                      int decode, void* O, int32_t* trace, const float* wpart, cudaStream_t s) {
  constexpr int D = 64 * NP;
  const int64_t kk = p.k < p.cap ? p.k : p.cap;
  int64_t maxn = 1;
  for (int l = 0; l < p.lay.levels; ++l) maxn = p.lay.nodes[l] > maxn ? p.lay.nodes[l] : maxn;
  int64_t cm = p.b * kk + p.b - 1;
  cm = cm < maxn ? cm : maxn;
  const int cmax = int(cm < 1 ? 1 : cm);
  if (cmax > kZMaxCand) return cudaErrorNotSupported;   // the generic kernel serves it
  const int kmax = int(kk < cmax ? kk : cmax);
  const bool part = wpart != nullptr;   // prefill with window partials: small CTAs
  const int nch = part ? kZPreChain : kZDecChain, nw = part ? kZPreChain : kZDecChain + kZDecWin;
  // level key rows staged per chunk (FP8 rows are a quarter of the bytes, NVFP4
  // rows less); small CTAs keep their staging to 40 KB so that four share an SM
  const bool lowp = p.kfmt != RECSA_KEYS_F32;
  const int rowb = p.kfmt == RECSA_KEYS_FP8 ? D : (lowp ? D / 2 + D / 16 : 4 * D);
  const size_t stage = part ? 40 * 1024 : kZStageBytes;
  const int krows = int(std::min<int64_t>(int64_t(cmax) * p.nref, int64_t(stage / size_t(rowb + 8))));
  if (krows < p.nref) return cudaErrorNotSupported;
  const int rounds = (cmax + nch * 32 - 1) / (nch * 32);
  const size_t bytes = size_t(krows) * rowb +
                       (2 * size_t(krows) + 2 * size_t(cmax) + nch + 1 + size_t(nw) * (D + 2)) * 4 +
                       (2 * size_t(kmax) + 2 * (kMaxLevels + 1) + size_t(cmax) +
                        size_t(rounds) * nch) * 4;
  if (bytes > 227 * 1024) return cudaErrorNotSupported;
  if (p.batch > 65535) return cudaErrorNotSupported;
  auto kern = part ? zha_attend_kernel<T, NP, kZPreChain, 0>
                   : zha_attend_kernel<T, NP, kZDecChain, kZDecWin>;
  cudaError_t e = ensure_smem(kern, int(bytes));
  if (e != cudaSuccess) return e;
  dim3 grid(n_q, p.batch, p.hq);
  kern<<<grid, nw * 32, bytes, s>>>(p, reinterpret_cast<const T*>(Q),
                                    reinterpret_cast<const T*>(K),
                                    reinterpret_cast<const T*>(V), tree, len_dev, q_start, n_q,
                                    decode, reinterpret_cast<T*>(O), trace, cmax, kmax, krows,
                                    wpart);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_zha(const Params& p, const void* Q, const void* K, const void* V,
                       const void* tree, const int64_t* len_dev, int64_t q_start, int32_t n_q,
                       int decode, void* O, int32_t* trace, const void* wpart, cudaStream_t s) {
  if (p.mode != RECSA_MODE_ZHA) return cudaErrorNotSupported;
  const float* wp = decode ? nullptr : reinterpret_cast<const float*>(wpart);
  if (p.dtype == RECSA_DTYPE_BF16)
    return p.d == 128 ? zha_typed<__nv_bfloat16, 2>(p, Q, K, V, tree, len_dev, q_start, n_q,
                                                    decode, O, trace, wp, s)
                      : zha_typed<__nv_bfloat16, 1>(p, Q, K, V, tree, len_dev, q_start, n_q,
                                                    decode, O, trace, wp, s);
  return p.d == 128 ? zha_typed<float, 2>(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O,
                                          trace, wp, s)
                    : zha_typed<float, 1>(p, Q, K, V, tree, len_dev, q_start, n_q, decode, O,
                                          trace, wp, s);
}

}  // namespace recsa
