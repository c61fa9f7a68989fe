// Attention on 5th-generation tensor cores (tcgen05 + TMEM + TMA), shared by
//   K2  compressed branch with the fused streaming top-k of S_guide
//       ("Speed3R: Sparse Feed-forward 3D Reconstruction Models", Paper-Notes
//       CVPR 2026, compression branch; "高效 Triton Kernel 实现": top-k kept
//       while the FlashAttention loop runs, S_guide never materialised);
//   K5  special tokens over every token (split over key ranges, merged later);
//   K6  dense global attention (the comparison baseline).
//
// One CTA owns two 128-row query tiles (M = 256) that share every K/V tile, so
// each key byte crosses L2 -> SM once per 256 queries.  Warp roles:
//   warps 0-3  softmax for query tile 0 (thread = row = TMEM lane)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q tiles once, then K/V tiles into a 3-stage ring
//   warp  9    MMA issuer (one thread): S_i = Q_i K^T (SS form, both operands
//              in 128B-swizzled shared memory) and O_i += P_i V (TS form: P_i
//              read from TMEM, V as an MN-major shared-memory operand)
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,320), O_1 [320,384),
// P_0 [384,448), P_1 [448,512) (bf16 pairs).
// Softmax threads read their row of S_i, write P_i (bf16 pairs) to its own
// TMEM columns, and rescale O_i in TMEM only when the running max grows by
// more than 2^8 (lazy rescaling: the stale max keeps every exponent <= 2^8,
// and numerator and denominator share it).  The two softmax warpgroups run
// their exponentials at the same time: with two warps per SM sub-partition
// feeding the MUFU, one warp's non-MUFU instructions and dependency stalls
// are covered by the other's exponentials.
//
// Guide scores (K2): Q and K arrive as bf16 pairs hi + lo (lo = bf16 of the
// residual), S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T, accurate to ~2^-17 of
// |q||k|, so the top-k agrees with exact scores wherever the k-th and
// (k+1)-th scores differ by more than a few 1e-5 relative.  The streaming
// top-k is a sorted register list per thread (its row): a score strictly
// greater than the current k-th enters by an unrolled shift network; keys
// arrive in increasing region order, so on equal scores the lower region
// stays ahead, as the tie rule requires.
//
// All mbarrier waits are bounded by the global timer; a wait that runs out
// records GSA_ERR_DEVICE_TIMEOUT and the CTA drains and exits.
#include <cuda.h>

#include "gsa_kernels.h"
#include "tc_ptx.cuh"

namespace gsa {

namespace {

using namespace tc;

constexpr int TBM = 128;                 // rows per query tile
constexpr int TBN = 128;                 // keys per tile
constexpr int TILE = TBN * 128;          // bytes of one 128x64 bf16 tile
constexpr int NTHREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.f;      // rescale O when the max grows by > 2^8

constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 64, true);

// GO (guide only, the "no compressed value" ablation): S and the top-k, no P V.
template <int KC, bool GO = false>
struct Lay {
  static constexpr bool TOPK = KC > 0;
  static constexpr int NST = 3;                        // K/V ring depth
  static constexpr int QT = TOPK ? 2 : 1;              // tiles per query tile (hi[, lo])
  static constexpr int KT = GO ? 2 : (TOPK ? 3 : 2);   // tiles per stage: K hi, [K lo], [V]
  static constexpr int KV = 2 * QT * TILE;             // Q_i hi at i*TILE, lo at (2+i)*TILE
  static constexpr int STAGE = KT * TILE;
  static constexpr int BAR = KV + NST * STAGE;
  // barriers: q_full, full[NST], empty[NST], s_full[2], s_free[2], p_full[2], pv_done[2], fin
  static constexpr int NBAR = 1 + 2 * NST + 8 + 1;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int BYTES = TMEM_SLOT + 16 + 1024;   // + alignment slack
};

struct Bars {
  uint32_t base;
  int nst;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t full(int s) const { return base + 8 * (1 + s); }
  __device__ uint32_t empty(int s) const { return base + 8 * (1 + nst + s); }
  __device__ uint32_t s_full(int i) const { return base + 8 * (1 + 2 * nst + i); }
  __device__ uint32_t s_free(int i) const { return base + 8 * (3 + 2 * nst + i); }
  __device__ uint32_t p_full(int i) const { return base + 8 * (5 + 2 * nst + i); }
  __device__ uint32_t pv_done(int i) const { return base + 8 * (7 + 2 * nst + i); }
  __device__ uint32_t fin() const { return base + 8 * (9 + 2 * nst); }
};

// one arrival per warp, after every lane's preceding work (fences included)
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ int tile_seg(const AttnArgs& a, int tt, long long& kb) {
  const int seg = (a.nseg > 1 && tt >= a.tiles0) ? 1 : 0;
  kb = static_cast<long long>(seg ? tt - a.tiles0 : tt) * TBN;
  return seg;
}


// validity bits of a 128-key tile, one word per 32-key chunk (bit e of word c
// = key kb + 32c + e).  A frame is `lead` always-valid keys (its special tokens,
// dense layout only) and then Hp rows of Wp slots whose first Wv slots of the
// first Hv rows are valid.  One division places the tile's first key in its
// frame; the tile is then walked run by run (a valid stretch of a grid row, its
// pad columns, the pad rows, the lead), the position advancing without division.
__device__ __noinline__ uint4 tile_valid(int km, Grid g, int nk, long long kb) {
  uint32_t w[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const long long lim = nk - kb - 32 * c;
    w[c] = lim >= 32 ? ~0u : (lim <= 0 ? 0u : ((1u << lim) - 1u));
  }
  if (km != MASK_NONE && w[0] != 0u) {
    const int lead = km == MASK_DENSE ? g.ns : 0;
    const int per = lead + g.Hp * g.Wp;
    int o = static_cast<int>(kb) % per;          // kb < nk: a key index of one head
    int y = 0, x = 0;
    if (o >= lead) {
      y = (o - lead) / g.Wp;
      x = (o - lead) - y * g.Wp;
    }
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t v = 0;
      for (int e = 0; e < 32;) {
        int run;
        bool ok;
        const bool in_rows = o >= lead && y < g.Hv;
        if (o < lead) {
          run = lead - o;
          ok = true;
        } else if (y >= g.Hv) {
          run = per - o;                        // pad rows up to the end of the frame
          ok = false;
        } else if (x < g.Wv) {
          run = g.Wv - x;
          ok = true;
        } else {
          run = g.Wp - x;
          ok = false;
        }
        const int n = min(run, 32 - e);
        if (ok) v |= (n >= 32 ? ~0u : ((1u << n) - 1u)) << e;
        e += n;
        o += n;
        if (o >= per) {
          o = 0;                                // next frame
          y = 0;
          x = 0;
        } else if (in_rows) {
          x += n;                               // n <= Wp - x
          if (x >= g.Wp) {
            x = 0;
            ++y;
          }
        }
      }
      w[c] &= v;
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// c ? a : b through an explicit selp, so that chains of these over a
// register array stay register selects (never an indexed local-memory load)
__device__ __forceinline__ uint32_t sel_if(bool c, uint32_t a, uint32_t b) {
  uint32_t r;
  asm("{\n .reg .pred p;\n setp.ne.u32 p, %3, 0;\n selp.b32 %0, %1, %2, p;\n}\n"
      : "=r"(r)
      : "r"(a), "r"(b), "r"(static_cast<uint32_t>(c)));
  return r;
}

// v[e] for a runtime e in [0, 64): the first level folds bits 5 and 4 (four
// inputs per output, 16 live temporaries), then four levels of selects
__device__ __forceinline__ uint32_t pick64(const uint32_t* v, int e) {
  uint32_t t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    t[i] = sel_if(e & 32, sel_if(e & 16, v[i + 48], v[i + 32]), sel_if(e & 16, v[i + 16], v[i]));
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = sel_if(e & 8, t[i + 8], t[i]);
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = sel_if(e & 4, t[i + 4], t[i]);
#pragma unroll
  for (int i = 0; i < 2; ++i) t[i] = sel_if(e & 2, t[i + 2], t[i]);
  return sel_if(e & 1, t[1], t[0]);
}

// Two exponentials of the softmax with packed fp32x2 arithmetic (one FFMA2
// for both arguments, one FADD2 for both running sums): half the FMA-pipe
// issue slots of the scalar form, and exactly its roundings.
__device__ __forceinline__ void exp2_pair(uint32_t s0, uint32_t s1, float sl2, float nmb, float& l0, float& l1,
                                          float& p0, float& p1) {
  float x0, x1;
  asm("{\n .reg .b64 a, b, c, d;\n"
      " mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %4};\n mov.b64 c, {%5, %5};\n"
      " fma.rn.f32x2 d, a, b, c;\n mov.b64 {%0, %1}, d;\n}\n"
      : "=f"(x0), "=f"(x1)
      : "r"(s0), "r"(s1), "f"(sl2), "f"(nmb));
  p0 = ex2(x0);
  p1 = ex2(x1);
  asm("{\n .reg .b64 a, b;\n"
      " mov.b64 a, {%0, %1};\n mov.b64 b, {%2, %3};\n add.rn.f32x2 a, a, b;\n mov.b64 {%0, %1}, a;\n}\n"
      : "+f"(l0), "+f"(l1)
      : "f"(p0), "f"(p1));
}

// max of 32 values with 4 independent chains
__device__ __forceinline__ float max32(const uint32_t* v) {
  float m0 = __uint_as_float(v[0]), m1 = __uint_as_float(v[1]), m2 = __uint_as_float(v[2]),
        m3 = __uint_as_float(v[3]);
#pragma unroll
  for (int e = 4; e < 32; e += 4) {
    m0 = fmaxf(m0, __uint_as_float(v[e]));
    m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
    m2 = fmaxf(m2, __uint_as_float(v[e + 2]));
    m3 = fmaxf(m3, __uint_as_float(v[e + 3]));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

__device__ __forceinline__ void apply_mask(uint32_t* v, uint32_t msk) {
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = ((msk >> e) & 1u) ? v[e] : 0xff800000u;   // -inf
}

// bits of the 32 regions col0 .. col0 + 31 that lie in fixed-context frames
// (never top-k candidates)
__device__ __forceinline__ uint32_t fixed_bits(const AttnArgs& a, int col0) {
  uint32_t b = 0;
  for (int f = 0; f < a.n_fixed; ++f) {
    const int lo = max(a.fixed[f] * a.rpf - col0, 0);
    const int hi = min((a.fixed[f] + 1) * a.rpf - col0, 32);
    if (hi > lo) b |= (hi - lo >= 32 ? ~0u : ((1u << (hi - lo)) - 1u)) << lo;
  }
  return b;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Lazy rescale: move the reference max only when the row max grew by more than
// 2^8; O_i (in TMEM) is rescaled once PV of the previous tile has completed.
// The decision to touch TMEM is warp-uniform (TMEM loads are warp-collective).
template <int PIECE>
__device__ __forceinline__ void rescale(float mx, float& m, float& l, int j, int qi, uint32_t tO,
                                        const Bars& bars, int* err, bool& ok, float sl2) {
  const float m_new = fmaxf(m, mx);
  const bool need = (m == -INFINITY) ? (m_new != -INFINITY) : ((m_new - m) * sl2 > RESCALE_LOG2);
  float alpha = 1.f;
  if (need) {
    alpha = (m == -INFINITY) ? 0.f : ex2((m - m_new) * sl2);
    m = m_new;
  }
  l *= alpha;
  if (__any_sync(0xffffffffu, need && alpha != 0.f) && j > 0) {
    ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(qi), (j - 1) & 1, err));
    if (!ok) return;
    tc_fence_after();
    if constexpr (PIECE == 8) {
      // eight columns at a time: the caller holds a half-row of S and its top-k list
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t w[8];
        tmem_ld8(tO + 8 * c, w);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
        tmem_st8(tO + 8 * c, w);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t w[32];
        tmem_ld32(tO + 32 * c, w);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
        tmem_st32(tO + 32 * c, w);
      }
    }
    tmem_wait_st();
  }
}

// current k-th score of the list (the list may be longer than the run's k)
template <int KC>
__device__ __forceinline__ float kth_score(const float (&ts)[KC > 0 ? KC : 1], int kc) {
  if (kc == KC) return ts[KC - 1];
  uint32_t t = __float_as_uint(ts[KC - 1]);
#pragma unroll
  for (int p = 0; p < KC; ++p) t = sel_if(p == kc - 1, __float_as_uint(ts[p]), t);
  return __uint_as_float(t);
}

template <int KC>
__device__ __forceinline__ void topk_insert(float (&ts)[KC > 0 ? KC : 1], int (&ti)[KC > 0 ? KC : 1],
                                            float s, int id) {
  bool h = s > ts[KC - 1];
#pragma unroll
  for (int p = KC - 1; p > 0; --p) {
    const bool g = s > ts[p - 1];
    ts[p] = g ? ts[p - 1] : (h ? s : ts[p]);
    ti[p] = g ? ti[p - 1] : (h ? id : ti[p]);
    h = g;
  }
  if (h) {
    ts[0] = s;
    ti[0] = id;
  }
}

// MP (top-k beyond one 32-entry list): 0 a single pass; 1 the first of several
// passes; 2 a later pass, in which columns at or ahead of the previous pass's last
// selection (a.excl_s / a.excl_i) in the order (score desc, index asc) are not
// candidates, so the pass continues the sorted selection.  Passes 1 and 2 write
// their last selection (a.last_s / a.last_i) when asked.
template <int KC, bool GO, int MP = 0>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qlo,
                   const __grid_constant__ CUtensorMap tm_k0, const __grid_constant__ CUtensorMap tm_v0,
                   const __grid_constant__ CUtensorMap tm_k1, const __grid_constant__ CUtensorMap tm_v1,
                   const __grid_constant__ CUtensorMap tm_klo, const AttnArgs a) {
  using L = Lay<KC, GO>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const Bars bars{sbase + L::BAR, L::NST};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + L::TMEM_SLOT);

  const int warp = threadIdx.x >> 5;
  const int h = blockIdx.z, split = blockIdx.y;
  const int row0 = blockIdx.x * (2 * TBM);
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(t_begin + a.tiles_per_split, a.tiles_total);
  const int ntile = max(t_end - t_begin, 0);

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < L::NST; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.s_free(i), TBM / 32);     // one arrival per softmax warp
      mbar_init(bars.p_full(i), TBM / 32);
      mbar_init(bars.pv_done(i), 1);
    }
    mbar_init(bars.fin(), 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc<TMEM_COLS>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (ntile > 0) {
      const bool leader = elect_one();
      const int qy = h * a.n_q + row0;
      if (leader) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k0);
        prefetch_tmap(&tm_v0);
        mbar_expect_tx(bars.q_full(), 2 * L::QT * TILE);
        tma_load_2d(sbase + 0 * TILE, &tm_q, 0, qy, bars.q_full());
        tma_load_2d(sbase + 1 * TILE, &tm_q, 0, qy + TBM, bars.q_full());
        if constexpr (L::TOPK) {
          tma_load_2d(sbase + 2 * TILE, &tm_qlo, 0, qy, bars.q_full());
          tma_load_2d(sbase + 3 * TILE, &tm_qlo, 0, qy + TBM, bars.q_full());
        }
      }
      __syncwarp();
      int issued = 0;
      for (int it = 0; it < ntile; ++it) {
        const int s = it % L::NST;
        if (it >= L::NST &&
            !__all_sync(0xffffffffu, mbar_wait(bars.empty(s), ((it / L::NST) - 1) & 1, a.err)))
          break;
        long long kb;
        const int seg = tile_seg(a, t_begin + it, kb);
        const int y = static_cast<int>(static_cast<long long>(h) * a.n_k[seg] + kb);
        const uint32_t st = sbase + L::KV + s * L::STAGE;
        if (leader) {
          mbar_expect_tx(bars.full(s), L::KT * TILE);
          tma_load_2d(st, seg ? &tm_k1 : &tm_k0, 0, y, bars.full(s));
          if constexpr (L::TOPK) tma_load_2d(st + TILE, &tm_klo, 0, y, bars.full(s));
          if constexpr (!GO) tma_load_2d(st + (L::KT - 1) * TILE, seg ? &tm_v1 : &tm_v0, 0, y, bars.full(s));
        }
        __syncwarp();
        ++issued;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int it = max(0, issued - L::NST); it < issued; ++it)
        mbar_wait(bars.full(it % L::NST), (it / L::NST) & 1, a.err);
      mbar_wait(bars.q_full(), 0, a.err);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (operands stay warp-uniform); one elected
    // lane issues every MMA and commit.  Descriptors are built once and
    // advanced by adding to their start-address field (16-byte units).
    if (ntile > 0) {
      const bool leader = elect_one();
      const uint64_t dq0 = sdesc_sw128(sbase, 16, 1024);                    // Q_0 hi
      const uint64_t dk0 = sdesc_sw128(sbase + L::KV, 16, 1024);            // stage 0 K hi
      const uint64_t dv0 = sdesc_sw128(sbase + L::KV + (L::KT - 1) * TILE, 8192, 1024);   // stage 0 V
      constexpr uint32_t T16 = TILE >> 4, ST16 = L::STAGE >> 4;
      bool ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), 0, a.err));
      tc_fence_after();
      for (int j = 0; ok && j <= ntile; ++j) {
        if (j < ntile) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.full(j % L::NST), (j / L::NST) & 1, a.err));
          if (!ok) break;
          tc_fence_after();
        }
        const uint64_t dk = dk0 + (j % L::NST) * ST16;
        const uint64_t dv = dv0 + ((j + L::NST - 1) % L::NST) * ST16;
        for (int i = 0; i < 2 && ok; ++i) {
          if (j < ntile) {
            // S_{i,j} = Q_i K_j^T (guide: + Q_i^hi K_j^lo + Q_i^lo K_j^hi), as soon as
            // warpgroup i has read S_{i,j-1} into registers
            if (j > 0) {
              ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(i), (j - 1) & 1, a.err));
              if (!ok) break;
              tc_fence_after();
            }
            const uint64_t dq = dq0 + i * T16;
            if (leader) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                mma_bf16_ss(tmem + 128 * i, dq + 2 * ks, dk + 2 * ks, IDESC_QK, ks > 0 ? 1u : 0u);
                if constexpr (L::TOPK) {
                  mma_bf16_ss(tmem + 128 * i, dq + 2 * ks, dk + T16 + 2 * ks, IDESC_QK, 1u);
                  mma_bf16_ss(tmem + 128 * i, dq + 2 * T16 + 2 * ks, dk + 2 * ks, IDESC_QK, 1u);
                }
              }
              mma_commit(bars.s_full(i));
            }
            __syncwarp();
          }
          if (!GO && j > 0) {
            // O_i += P_{i,j-1} V_{j-1}: P read from TMEM (TS form), V MN-major
            ok = __all_sync(0xffffffffu, mbar_wait(bars.p_full(i), (j - 1) & 1, a.err));
            if (!ok) break;
            tc_fence_after();
            if (leader) {
#pragma unroll
              for (int ks = 0; ks < TBN / 16; ++ks)
                mma_bf16_ts(tmem + 256 + 64 * i, tmem + 384 + 64 * i + 8 * ks, dv + ks * 128, IDESC_PV,
                            (j > 1 || ks > 0) ? 1u : 0u);
              mma_commit(bars.pv_done(i));
            }
            __syncwarp();
          }
        }
        if (ok && j > 0 && leader) mma_commit(bars.empty((j - 1) % L::NST));
        __syncwarp();
      }
      if (leader) mma_commit(bars.fin());
      __syncwarp();
      mbar_wait(bars.fin(), 0, a.err);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int qi = warp >> 2;                         // query tile 0 or 1
    const int r = threadIdx.x & 127;                  // row in the tile = TMEM lane
    const int row = row0 + qi * TBM + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * qi;
    const uint32_t tO = tmem + lane_off + 256 + 64 * qi;
    const uint32_t tP = tmem + lane_off + 384 + 64 * qi;
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    float ts[KC > 0 ? KC : 1], thr = -INFINITY;
    int ti[KC > 0 ? KC : 1];
#pragma unroll
    for (int p = 0; p < (KC > 0 ? KC : 1); ++p) {
      ts[p] = -INFINITY;
      ti[p] = -1;
    }
    bool ok = true;
    float ex_s = INFINITY;                            // MP 2: the previous pass's last selection
    int ex_i = -1;
    if constexpr (MP == 2) {
      if (row < a.n_q) {
        ex_s = a.excl_s[static_cast<long long>(h) * a.n_q + row];
        ex_i = a.excl_i[static_cast<long long>(h) * a.n_q + row];
      }
    }
    for (int j = 0; j < ntile; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full(qi), j & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      long long kb;
      const int seg = tile_seg(a, t_begin + j, kb);
      const int nk = a.n_k[seg];
      const int km = a.kmask[seg];
      // key validity of the tile's four 32-key chunks (all ones unless ragged or
      // padded): from the segment's table when it has one (first used after the
      // TMEM load of S, which covers the load's latency), else walked here
      uint32_t vm[4] = {~0u, ~0u, ~0u, ~0u};
      if (km != MASK_NONE || kb + TBN > nk) {
        uint4 t4;
        if constexpr (L::TOPK) {
          t4 = tile_valid(km, a.g, nk, kb);           // regions: only a ragged last tile
        } else {
          const uint32_t* kbits = seg ? a.kbits[1] : a.kbits[0];
          t4 = kbits ? __ldg(reinterpret_cast<const uint4*>(kbits) + (kb >> 7)) : tile_valid(km, a.g, nk, kb);
        }
        vm[0] = t4.x; vm[1] = t4.y; vm[2] = t4.z; vm[3] = t4.w;
      }
      float mx = -INFINITY;
      if constexpr (!L::TOPK) {
        // whole row of S in registers: one TMEM wait per tile, and S_i is handed
        // back to the MMA warp at once so S_{i,j+1} overlaps this tile's softmax
        uint32_t v[128];
        tmem_ld64(tS, v);
        tmem_ld64(tS + 64, v + 64);
        tmem_wait_ld();
        tc_fence_before();
        warp_arrive(bars.s_free(qi));
        float cm[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (vm[c] != ~0u) apply_mask(v + 32 * c, vm[c]);
          cm[c] = max32(v + 32 * c);
        }
        mx = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
        rescale<32>(mx, m, l, j, qi, tO, bars, a.err, ok, sl2);
        if (!ok) break;
        // P_i is free once PV of the previous tile has completed
        if (j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(qi), (j - 1) & 1, a.err));
          if (!ok) break;
        }
        const float mb = (m == -INFINITY) ? 0.f : m * sl2;
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float p0, p1;
            exp2_pair(v[32 * c + e], v[32 * c + e + 1], sl2, -mb, l0, l1, p0, p1);
            pk[e >> 1] = pack_bf16(p0, p1);
          }
          tmem_st16(tP + 16 * c, pk);
        }
        l += l0 + l1;
      } else {
        // One pass over two 64-key halves.  Each half: row max and the streaming
        // top-k, then (unless guide only) its part of the online softmax, so S_i
        // is read once and handed back to the MMA warp as soon as its second
        // half is in registers: S_{i,j+1} then overlaps most of this tile.
        float l0 = 0.f, l1 = 0.f;
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t v[64];
          tmem_ld64(tS + 64 * hf, v);
          tmem_wait_ld();
          if (hf == 1) {
            tc_fence_before();
            warp_arrive(bars.s_free(qi));
          }
          uint32_t cb[2] = {0u, 0u};
          float hmx = -INFINITY;
          float cmx[2];
          bool notmax[2] = {false, false};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t msk = sel_if(hf, vm[2 + c], vm[c]);
            if (msk != ~0u) apply_mask(v + 32 * c, msk);
            const float cmax = max32(v + 32 * c);
            cmx[c] = cmax;
            hmx = fmaxf(hmx, cmax);
            if (cmax > thr) {
#pragma unroll
              for (int e = 0; e < 32; ++e) cb[c] |= (__uint_as_float(v[32 * c + e]) > thr ? 1u : 0u) << e;
              if (a.n_fixed) {
                // fixed-context regions are never candidates; if one of them held
                // the chunk max, the max is no longer a candidate's value
                const uint32_t fb = fixed_bits(a, static_cast<int>(kb) + 64 * hf + 32 * c);
                notmax[c] = (cb[c] & fb) != 0u;
                cb[c] &= ~fb;
              }
              if constexpr (MP == 2) {
                if (cmax >= ex_s) {
                  // an earlier pass took these: score above its last, or equal at a lower index
                  const int col0 = static_cast<int>(kb) + 64 * hf + 32 * c;
#pragma unroll 1
                  for (int e = 0; e < 32; ++e) {
                    const float x = __uint_as_float(v[32 * c + e]);
                    if (x > ex_s || (x == ex_s && col0 + e <= ex_i)) cb[c] &= ~(1u << e);
                  }
                  notmax[c] = true;
                }
              }
            }
          }
          // rare: a score beats the current k-th; take the candidates in column
          // order through one insertion site for the whole half.  A chunk with a
          // single candidate needs no select tree: the candidate is the chunk max.
          const bool one0 = __popc(cb[0]) == 1 && !notmax[0], one1 = __popc(cb[1]) == 1 && !notmax[1];
          while (cb[0] | cb[1]) {
            const bool lo = cb[0] != 0;
            const int e = lo ? __ffs(cb[0]) - 1 : 31 + __ffs(cb[1]);
            if (lo) cb[0] &= cb[0] - 1; else cb[1] &= cb[1] - 1;
            const float x = (lo ? one0 : one1) ? (lo ? cmx[0] : cmx[1]) : __uint_as_float(pick64(v, e));
            const int col = static_cast<int>(kb) + 64 * hf + e;
            if (!(x > thr)) continue;
            topk_insert<KC>(ts, ti, x, col);
            thr = kth_score<KC>(ts, a.kc);
          }
          if constexpr (!GO) {
            // online softmax per half: the reference max moves only when this
            // half raises a row's max by more than 2^8 (rare after the first tile)
            const bool grow = (m == -INFINITY) ? (hmx != -INFINITY) : ((hmx - m) * sl2 > RESCALE_LOG2);
            if (__any_sync(0xffffffffu, grow)) {
              l += l0 + l1;
              l0 = l1 = 0.f;
              const float m_old = m;
              rescale<8>(hmx, m, l, j, qi, tO, bars, a.err, ok, sl2);
              if (!ok) break;
              if (hf == 1) {
                // P of the first half was written against the old max: scale it too
                const float alpha = (m == m_old) ? 1.f : (m_old == -INFINITY ? 0.f : ex2((m_old - m) * sl2));
                tmem_wait_st();
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                  uint32_t w[8];
                  tmem_ld8(tP + 8 * q, w);
                  tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
                    w[e] = pack_bf16(__low2float(b) * alpha, __high2float(b) * alpha);
                  }
                  tmem_st8(tP + 8 * q, w);
                }
              }
            }
            // P_i is free once PV of the previous tile has completed
            if (hf == 0 && j > 0) {
              ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(qi), (j - 1) & 1, a.err));
              if (!ok) break;
            }
            const float mb = (m == -INFINITY) ? 0.f : m * sl2;
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              float p0, p1;
              exp2_pair(v[e], v[e + 1], sl2, -mb, l0, l1, p0, p1);
              pk[e >> 1] = pack_bf16(p0, p1);
            }
            tmem_st32(tP + 32 * hf, pk);
          }
        }
        if (!ok) break;
        if constexpr (GO) continue;      // guide only: nothing else to compute
        l += l0 + l1;
      }
      tmem_wait_st();          // P (and any O rescale) written to TMEM
      tc_fence_before();
      warp_arrive(bars.p_full(qi));
    }
    // ---- epilogue: O_i row from TMEM ----------------------------------------
    if (!GO && ok && ntile > 0) ok = mbar_wait(bars.pv_done(qi), (ntile - 1) & 1, a.err);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    float o[64];
    if (!GO && ok && ntile > 0) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[32 * c + e] = __uint_as_float(v[e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 64; ++e) o[e] = 0.f;
    }
    if (row < a.n_q) {
      if (GO) {
        // guide only: no attention output
      } else if (a.n_split == 1) {
        if (a.lse) a.lse[static_cast<long long>(h) * a.n_q + row] = l > 0.f ? m * sl2 + __log2f(l) : -INFINITY;
        float inv = l > 0.f ? 1.f / l : 0.f;
        if (a.q_mask != MASK_NONE && !key_valid(a.q_mask, a.g, row)) inv = 0.f;
        const long long base = h * a.o_hs + static_cast<long long>(row) * D;
        if (a.o16) {
#pragma unroll
          for (int e = 0; e < 64; e += 8) {
            const uint4 w = make_uint4(pack_bf16(o[e] * inv, o[e + 1] * inv), pack_bf16(o[e + 2] * inv, o[e + 3] * inv),
                                       pack_bf16(o[e + 4] * inv, o[e + 5] * inv), pack_bf16(o[e + 6] * inv, o[e + 7] * inv));
            *reinterpret_cast<uint4*>(a.o16 + base + e) = w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; e += 4)
            *reinterpret_cast<float4*>(a.o32 + base + e) =
                make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
        }
      } else {
        const long long pr = (static_cast<long long>(split) * a.H + h) * a.n_q + row;
#pragma unroll
        for (int e = 0; e < 64; e += 4)
          *reinterpret_cast<float4*>(a.part_o + pr * D + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        *reinterpret_cast<float2*>(a.part_ml + pr * 2) = make_float2(m, l);
      }
      if constexpr (L::TOPK) {
        const long long base = MP == 0 ? (static_cast<long long>(h) * a.n_q + row) * a.kc
                                       : (static_cast<long long>(h) * a.n_q + row) * a.cand_stride + a.cand_off;
#pragma unroll
        for (int p = 0; p < KC; ++p) {
          if (p < a.kc) {
            a.cand[base + p] = ti[p];
            if (a.cand_user) a.cand_user[base + p] = ti[p];
          }
        }
        if (MP != 0 && a.last_s) {
          // the last selection of this pass, where the next pass continues
          a.last_s[static_cast<long long>(h) * a.n_q + row] = kth_score<KC>(ts, a.kc);
          int li = ti[KC - 1];
#pragma unroll
          for (int p = 0; p < KC; ++p) li = p == a.kc - 1 ? ti[p] : li;
          a.last_i[static_cast<long long>(h) * a.n_q + row] = li;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc<TMEM_COLS>(tmem);
}

// ---- tensor maps ----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 tensor [rows][64] with 128-row, 128B-swizzled boxes
bool make_map(CUtensorMap* m, const void* base, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base || rows <= 0 || rows > 0x7fffffffLL) return false;
  const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KC, bool GO, int MP = 0>
cudaError_t launch_kc(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t st) {
  const int sm = Lay<KC, GO>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<KC, GO, MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_q + 2 * TBM - 1) / (2 * TBM), a.n_split, a.H);
  attn_tc_kernel<KC, GO, MP><<<grid, NTHREADS, sm, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], a);
  return cudaGetLastError();
}

template <int KC>
cudaError_t launch_kc2(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t st) {
  return a.guide_only ? launch_kc<KC, true>(a, maps, st) : launch_kc<KC, false>(a, maps, st);
}

// ==== attention backward on tcgen05: dQ ======================================
// Per CTA one 128-row query tile (thread = row = TMEM lane) against every key
// tile: S = Q K^T (the forward's split guide where it had one) and
// dP = dO V^T into TMEM, the softmax warps turn them into
// dS = P o (dP - D) with P = exp2(S * scale * log2 e - lse2) (bf16 pairs into
// TMEM), and dQ += dS K runs in the TS form with K as an MN-major operand.
// TMEM: S [0,128), dP [128,256), dQ [256,320), dS [320,384).
// Warps 0-3 softmax, warp 4 TMA producer, warp 5 MMA issuer.
constexpr int BW_NTHREADS = 192;

struct BwdTc {
  BwdArgs b;
  int tiles0;                  // 128-key tiles of segment 0
  int tiles_total;
  int tiles_per_split;         // dQ: key tiles per split (blockIdx.z)
  int n_split;                 // dQ: > 1 adds each split's part to a zeroed dq
  int* err;
};

template <bool SPLIT>
struct DqLay {
  static constexpr int NST = 3;
  static constexpr int QT = SPLIT ? 3 : 2;     // Q hi, [Q lo], dO
  static constexpr int KT = SPLIT ? 3 : 2;     // K hi, [K lo], V
  static constexpr int KV = QT * TILE;
  static constexpr int STAGE = KT * TILE;
  static constexpr int BAR = KV + NST * STAGE;
  // q_full, full[NST], empty[NST], s_full, s_free, ds_full, dq_done, fin
  static constexpr int NBAR = 1 + 2 * NST + 5;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int BYTES = TMEM_SLOT + 16 + 1024;
};

struct DqBars {
  uint32_t base;
  int nst;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t full(int s) const { return base + 8 * (1 + s); }
  __device__ uint32_t empty(int s) const { return base + 8 * (1 + nst + s); }
  __device__ uint32_t s_full() const { return base + 8 * (1 + 2 * nst); }
  __device__ uint32_t s_free() const { return base + 8 * (2 + 2 * nst); }
  __device__ uint32_t ds_full() const { return base + 8 * (3 + 2 * nst); }
  __device__ uint32_t dq_done() const { return base + 8 * (4 + 2 * nst); }
  __device__ uint32_t fin() const { return base + 8 * (5 + 2 * nst); }
};

__device__ __forceinline__ int bw_seg(const BwdTc& t, int tt, long long& kb) {
  const int seg = (t.b.nseg > 1 && tt >= t.tiles0) ? 1 : 0;
  kb = static_cast<long long>(seg ? tt - t.tiles0 : tt) * TBN;
  return seg;
}

// dS of two keys: P = exp2(s * sl2 - lse2) (packed FFMA2), dS = P (dP - D)
__device__ __forceinline__ uint32_t ds_pair(uint32_t s0, uint32_t s1, uint32_t dp0, uint32_t dp1, float sl2,
                                            float nlse, float nD) {
  float x0, x1;
  asm("{\n .reg .b64 a, b, c, d;\n"
      " mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %4};\n mov.b64 c, {%5, %5};\n"
      " fma.rn.f32x2 d, a, b, c;\n mov.b64 {%0, %1}, d;\n}\n"
      : "=f"(x0), "=f"(x1)
      : "r"(s0), "r"(s1), "f"(sl2), "f"(nlse));
  const float p0 = ex2(x0), p1 = ex2(x1);
  float d0, d1;
  asm("{\n .reg .b64 a, b, c, d;\n"
      " mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %4};\n add.rn.f32x2 c, a, b;\n"
      " mov.b64 d, {%5, %6};\n mul.rn.f32x2 c, c, d;\n mov.b64 {%0, %1}, c;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "r"(dp0), "r"(dp1), "f"(nD), "f"(p0), "f"(p1));
  return pack_bf16(d0, d1);
}

template <bool SPLIT>
__global__ void __launch_bounds__(BW_NTHREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qlo,
                          const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_k0,
                          const __grid_constant__ CUtensorMap tm_v0, const __grid_constant__ CUtensorMap tm_k1,
                          const __grid_constant__ CUtensorMap tm_v1, const __grid_constant__ CUtensorMap tm_klo,
                          const BwdTc t) {
  using L = DqLay<SPLIT>;
  const BwdArgs& a = t.b;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const DqBars bars{sbase + L::BAR, L::NST};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + L::TMEM_SLOT);
  const int warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int row0 = blockIdx.x * TBM;
  // this CTA's key tiles: split blockIdx.z of the key range
  const int t_begin = blockIdx.z * t.tiles_per_split;
  const int ntile = max(min(t.tiles_per_split, t.tiles_total - t_begin), 0);

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < L::NST; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.s_free(), TBM / 32);
    mbar_init(bars.ds_full(), TBM / 32);
    mbar_init(bars.dq_done(), 1);
    mbar_init(bars.fin(), 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc<TMEM_COLS>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (ntile > 0) {
      const bool leader = elect_one();
      const int qy = h * a.n_q + row0;
      if (leader) {
        mbar_expect_tx(bars.q_full(), L::QT * TILE);
        tma_load_2d(sbase, &tm_q, 0, qy, bars.q_full());
        if constexpr (SPLIT) tma_load_2d(sbase + TILE, &tm_qlo, 0, qy, bars.q_full());
        tma_load_2d(sbase + (L::QT - 1) * TILE, &tm_do, 0, qy, bars.q_full());
      }
      __syncwarp();
      int issued = 0;
      for (int it = 0; it < ntile; ++it) {
        const int s = it % L::NST;
        if (it >= L::NST &&
            !__all_sync(0xffffffffu, mbar_wait(bars.empty(s), ((it / L::NST) - 1) & 1, t.err)))
          break;
        long long kb;
        const int seg = bw_seg(t, t_begin + it, kb);
        const int y = static_cast<int>(static_cast<long long>(h) * a.n_k[seg] + kb);
        const uint32_t st = sbase + L::KV + s * L::STAGE;
        if (leader) {
          mbar_expect_tx(bars.full(s), L::KT * TILE);
          tma_load_2d(st, seg ? &tm_k1 : &tm_k0, 0, y, bars.full(s));
          if constexpr (SPLIT) tma_load_2d(st + TILE, &tm_klo, 0, y, bars.full(s));
          tma_load_2d(st + (L::KT - 1) * TILE, seg ? &tm_v1 : &tm_v0, 0, y, bars.full(s));
        }
        __syncwarp();
        ++issued;
      }
      for (int it = max(0, issued - L::NST); it < issued; ++it)
        mbar_wait(bars.full(it % L::NST), (it / L::NST) & 1, t.err);
      mbar_wait(bars.q_full(), 0, t.err);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (ntile > 0) {
      const bool leader = elect_one();
      constexpr uint32_t T16 = TILE >> 4, ST16 = L::STAGE >> 4;
      const uint64_t dq0 = sdesc_sw128(sbase, 16, 1024);                           // Q hi
      const uint64_t ddo = dq0 + (L::QT - 1) * T16;                               // dO
      const uint64_t dk0 = sdesc_sw128(sbase + L::KV, 16, 1024);                  // K hi, K-major
      const uint64_t dv0 = dk0 + (L::KT - 1) * T16;                               // V, K-major
      const uint64_t dkb0 = sdesc_sw128(sbase + L::KV, 8192, 1024);               // K hi, MN-major
      bool ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), 0, t.err));
      tc_fence_after();
      for (int j = 0; ok && j <= ntile; ++j) {
        if (j < ntile) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.full(j % L::NST), (j / L::NST) & 1, t.err));
          if (!ok) break;
          if (j > 0) ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (j - 1) & 1, t.err));
          if (!ok) break;
          tc_fence_after();
          const uint64_t dk = dk0 + (j % L::NST) * ST16, dv = dv0 + (j % L::NST) * ST16;
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              mma_bf16_ss(tmem, dq0 + 2 * ks, dk + 2 * ks, IDESC_QK, ks > 0 ? 1u : 0u);
              if constexpr (SPLIT) {
                mma_bf16_ss(tmem, dq0 + 2 * ks, dk + T16 + 2 * ks, IDESC_QK, 1u);
                mma_bf16_ss(tmem, dq0 + T16 + 2 * ks, dk + 2 * ks, IDESC_QK, 1u);
              }
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem + 128, ddo + 2 * ks, dv + 2 * ks, IDESC_QK, ks > 0 ? 1u : 0u);
            mma_commit(bars.s_full());
          }
          __syncwarp();
        }
        if (j > 0) {
          // dQ += dS_{j-1} K_{j-1}: dS read from TMEM (TS form), K MN-major
          ok = __all_sync(0xffffffffu, mbar_wait(bars.ds_full(), (j - 1) & 1, t.err));
          if (!ok) break;
          tc_fence_after();
          const uint64_t dkb = dkb0 + ((j - 1) % L::NST) * ST16;
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < TBN / 16; ++ks)
              mma_bf16_ts(tmem + 256, tmem + 320 + 8 * ks, dkb + ks * 128, IDESC_PV, (j > 1 || ks > 0) ? 1u : 0u);
            mma_commit(bars.dq_done());
            mma_commit(bars.empty((j - 1) % L::NST));
          }
          __syncwarp();
        }
      }
      if (leader) mma_commit(bars.fin());
      __syncwarp();
      mbar_wait(bars.fin(), 0, t.err);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                        // row in the tile = TMEM lane
    const int row = row0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off, tP = tS + 128, tQ = tS + 256, tD = tS + 320;
    const float sl2 = a.scale_log2;
    const bool rv = row < a.n_q;
    // rows past the end: lse = +inf makes P (and dS) zero
    const float nlse = rv ? -a.lse2[static_cast<long long>(h) * a.n_q + row] : -INFINITY;
    const float nD = rv ? -a.Dv[static_cast<long long>(h) * a.n_q + row] : 0.f;
    bool ok = true;
    for (int j = 0; j < ntile; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full(), j & 1, t.err));
      if (!ok) break;
      tc_fence_after();
      long long kb;
      const int seg = bw_seg(t, t_begin + j, kb);
      const int nk = a.n_k[seg];
      const int km = a.kmask[seg];
      uint32_t vm[4] = {~0u, ~0u, ~0u, ~0u};
      if (km != MASK_NONE || kb + TBN > nk) {
        const uint32_t* kbits = a.kbits[seg];
        const uint4 t4 = kbits ? __ldg(reinterpret_cast<const uint4*>(kbits) + (kb >> 7)) : tile_valid(km, a.g, nk, kb);
        vm[0] = t4.x; vm[1] = t4.y; vm[2] = t4.z; vm[3] = t4.w;
      }
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sv[64], pv[64];
        tmem_ld64(tS + 64 * hf, sv);
        tmem_ld64(tP + 64 * hf, pv);
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          warp_arrive(bars.s_free());
        }
        const uint32_t m0 = sel_if(hf, vm[2], vm[0]), m1 = sel_if(hf, vm[3], vm[1]);
        if (m0 != ~0u) apply_mask(sv, m0);
        if (m1 != ~0u) apply_mask(sv + 32, m1);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) pk[e >> 1] = ds_pair(sv[e], sv[e + 1], pv[e], pv[e + 1], sl2, nlse, nD);
        // dS_i is free once dQ of the previous tile has completed
        if (hf == 0 && j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.dq_done(), (j - 1) & 1, t.err));
          if (!ok) break;
        }
        tmem_st32(tD + 32 * hf, pk);
      }
      if (!ok) break;
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(bars.ds_full());
    }
    if (ok && ntile > 0) ok = mbar_wait(bars.dq_done(), (ntile - 1) & 1, t.err);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok && ntile > 0) {
      float* out = a.dq + h * a.dq_hs + static_cast<long long>(rv ? row : 0) * D;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t w[32];
        tmem_ld32(tQ + 32 * c, w);            // warp-collective: every lane loads
        tmem_wait_ld();
        if (rv) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v = make_float4(__uint_as_float(w[e]) * a.scale, __uint_as_float(w[e + 1]) * a.scale,
                                   __uint_as_float(w[e + 2]) * a.scale, __uint_as_float(w[e + 3]) * a.scale);
            float* p = out + 32 * c + e;
            if (t.n_split > 1) {
              // key splits: each adds its part (dq was zeroed by the launcher)
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "f"(v.x), "f"(v.y),
                           "f"(v.z), "f"(v.w)
                           : "memory");
            } else {
              if (a.dq_accum) {
                const float4 o = *reinterpret_cast<const float4*>(p);
                v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
              }
              *reinterpret_cast<float4*>(p) = v;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc<TMEM_COLS>(tmem);
}

template <bool SPLIT>
cudaError_t launch_dq_tc(const BwdTc& t, const CUtensorMap* maps, cudaStream_t st) {
  const int sm = DqLay<SPLIT>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  dim3 grid((t.b.n_q + TBM - 1) / TBM, t.b.H, t.n_split);
  attn_bwd_dq_tc_kernel<SPLIT><<<grid, BW_NTHREADS, sm, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                                                              maps[6], maps[7], t);
  return cudaGetLastError();
}

// ==== attention backward on tcgen05: dK, dV ==================================
// Per CTA one 128-key tile of one key segment (thread = key = TMEM lane)
// against every query tile: S^T = K Q^T (split guide where the forward had
// one) and dP^T = V dO^T into TMEM; the softmax warps form
// P^T = exp2(S^T * scale * log2 e - lse2[query]) and dS^T = P^T o (dP^T - D[query])
// in bf16 pairs; dV += P^T dO and dK += dS^T Q run in the TS form with dO and Q
// as MN-major operands.  lse2 and D of a query tile sit in shared memory next
// to its tiles (written by the producer warp).
// TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384),
// P^T [384,448), dS^T [448,512).
template <bool SPLIT>
struct DkvLay {
  static constexpr int NST = 3;
  static constexpr int KT = SPLIT ? 3 : 2;     // resident: K hi, [K lo], V
  static constexpr int QT = SPLIT ? 3 : 2;     // per stage: Q hi, [Q lo], dO
  static constexpr int KV = KT * TILE;
  static constexpr int LD = QT * TILE;         // -lse2[128] then -D[128] after the stage's tiles
  static constexpr int STAGE = QT * TILE + 1024;
  static constexpr int BAR = KV + NST * STAGE;
  // k_full, full[NST], empty[NST], s_full, s_free, pds_full, kv_done, fin
  static constexpr int NBAR = 1 + 2 * NST + 5;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int BYTES = TMEM_SLOT + 16 + 1024;
};

template <bool SPLIT>
__global__ void __launch_bounds__(BW_NTHREADS, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qlo,
                           const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_klo,
                           const BwdTc t, const int seg) {
  using L = DkvLay<SPLIT>;
  const BwdArgs& a = t.b;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const DqBars bars{sbase + L::BAR, L::NST};      // q_full() is the resident K/V tiles here
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + L::TMEM_SLOT);
  const int warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int key0 = blockIdx.x * TBM;
  const int nk = a.n_k[seg];
  const int ntile = (a.n_q + TBN - 1) / TBN;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < L::NST; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.s_free(), TBM / 32);
    mbar_init(bars.ds_full(), TBM / 32);
    mbar_init(bars.dq_done(), 1);
    mbar_init(bars.fin(), 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc<TMEM_COLS>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (ntile > 0) {
      const int lane = threadIdx.x & 31;
      const bool leader = elect_one();
      const int ky = h * nk + key0;
      if (leader) {
        mbar_expect_tx(bars.q_full(), L::KT * TILE);
        tma_load_2d(sbase, &tm_k, 0, ky, bars.q_full());
        if constexpr (SPLIT) tma_load_2d(sbase + TILE, &tm_klo, 0, ky, bars.q_full());
        tma_load_2d(sbase + (L::KT - 1) * TILE, &tm_v, 0, ky, bars.q_full());
      }
      __syncwarp();
      int issued = 0;
      for (int it = 0; it < ntile; ++it) {
        const int s = it % L::NST;
        if (it >= L::NST &&
            !__all_sync(0xffffffffu, mbar_wait(bars.empty(s), ((it / L::NST) - 1) & 1, t.err)))
          break;
        const uint32_t st = sbase + L::KV + s * L::STAGE;
        // -lse2 and -D of the tile's queries (rows past the end: P = 0)
        float* ld = reinterpret_cast<float*>(sgen + L::KV + s * L::STAGE + L::LD);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = it * TBN + 32 * q + lane;
          const bool ok = row < a.n_q;
          const long long gi = static_cast<long long>(h) * a.n_q + (ok ? row : 0);
          ld[32 * q + lane] = ok ? -a.lse2[gi] : -INFINITY;
          ld[TBN + 32 * q + lane] = ok ? -a.Dv[gi] : 0.f;
        }
        __syncwarp();
        const int y = h * a.n_q + it * TBN;
        if (leader) {
          mbar_expect_tx(bars.full(s), L::QT * TILE);
          tma_load_2d(st, &tm_q, 0, y, bars.full(s));
          if constexpr (SPLIT) tma_load_2d(st + TILE, &tm_qlo, 0, y, bars.full(s));
          tma_load_2d(st + (L::QT - 1) * TILE, &tm_do, 0, y, bars.full(s));
        }
        __syncwarp();
        ++issued;
      }
      for (int it = max(0, issued - L::NST); it < issued; ++it)
        mbar_wait(bars.full(it % L::NST), (it / L::NST) & 1, t.err);
      mbar_wait(bars.q_full(), 0, t.err);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (ntile > 0) {
      const bool leader = elect_one();
      constexpr uint32_t T16 = TILE >> 4, ST16 = L::STAGE >> 4;
      const uint64_t dk = sdesc_sw128(sbase, 16, 1024);                           // K hi (A)
      const uint64_t dvv = dk + (L::KT - 1) * T16;                                // V (A)
      const uint64_t dq0 = sdesc_sw128(sbase + L::KV, 16, 1024);                  // Q hi, K-major (B)
      const uint64_t ddo0 = dq0 + (L::QT - 1) * T16;                              // dO, K-major (B)
      const uint64_t dqm0 = sdesc_sw128(sbase + L::KV, 8192, 1024);               // Q hi, MN-major (B)
      const uint64_t ddom0 = dqm0 + (L::QT - 1) * T16;                            // dO, MN-major (B)
      bool ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), 0, t.err));
      tc_fence_after();
      for (int j = 0; ok && j <= ntile; ++j) {
        if (j < ntile) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.full(j % L::NST), (j / L::NST) & 1, t.err));
          if (!ok) break;
          if (j > 0) ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (j - 1) & 1, t.err));
          if (!ok) break;
          tc_fence_after();
          const uint64_t dq = dq0 + (j % L::NST) * ST16, ddo = ddo0 + (j % L::NST) * ST16;
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              mma_bf16_ss(tmem, dk + 2 * ks, dq + 2 * ks, IDESC_QK, ks > 0 ? 1u : 0u);
              if constexpr (SPLIT) {
                mma_bf16_ss(tmem, dk + T16 + 2 * ks, dq + 2 * ks, IDESC_QK, 1u);
                mma_bf16_ss(tmem, dk + 2 * ks, dq + T16 + 2 * ks, IDESC_QK, 1u);
              }
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem + 128, dvv + 2 * ks, ddo + 2 * ks, IDESC_QK, ks > 0 ? 1u : 0u);
            mma_commit(bars.s_full());
          }
          __syncwarp();
        }
        if (j > 0) {
          // dV += P^T dO, dK += dS^T Q of tile j-1 (TS form, dO and Q MN-major)
          ok = __all_sync(0xffffffffu, mbar_wait(bars.ds_full(), (j - 1) & 1, t.err));
          if (!ok) break;
          tc_fence_after();
          const uint64_t dqm = dqm0 + ((j - 1) % L::NST) * ST16, ddom = ddom0 + ((j - 1) % L::NST) * ST16;
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < TBN / 16; ++ks) {
              mma_bf16_ts(tmem + 256, tmem + 384 + 8 * ks, ddom + ks * 128, IDESC_PV, (j > 1 || ks > 0) ? 1u : 0u);
              mma_bf16_ts(tmem + 320, tmem + 448 + 8 * ks, dqm + ks * 128, IDESC_PV, (j > 1 || ks > 0) ? 1u : 0u);
            }
            mma_commit(bars.dq_done());
            mma_commit(bars.empty((j - 1) % L::NST));
          }
          __syncwarp();
        }
      }
      if (leader) mma_commit(bars.fin());
      __syncwarp();
      mbar_wait(bars.fin(), 0, t.err);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                        // key in the tile = TMEM lane
    const int key = key0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off, tP = tS + 128, tV = tS + 256, tK = tS + 320, tPT = tS + 384,
                   tDS = tS + 448;
    const float sl2 = a.scale_log2;
    const bool kv = key < nk && key_valid(a.kmask[seg], a.g, key);
    bool ok = true;
    for (int j = 0; j < ntile; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full(), j & 1, t.err));
      if (!ok) break;
      // the producer's lse2/D stores of this stage: acquired through its full barrier
      // (complete by now; the stage cannot be refilled before this tile's dK/dV MMAs)
      ok = __all_sync(0xffffffffu, mbar_wait(bars.full(j % L::NST), (j / L::NST) & 1, t.err));
      if (!ok) break;
      tc_fence_after();
      const float* ld = reinterpret_cast<const float*>(sgen + L::KV + (j % L::NST) * L::STAGE + L::LD);
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sv[64], pv[64];
        tmem_ld64(tS + 64 * hf, sv);
        tmem_ld64(tP + 64 * hf, pv);
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          warp_arrive(bars.s_free());
        }
        if (!kv) apply_mask(sv, 0u), apply_mask(sv + 32, 0u);
        uint32_t pk[32], dk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 nl = *reinterpret_cast<const float2*>(ld + 64 * hf + e);
          const float2 nd = *reinterpret_cast<const float2*>(ld + TBN + 64 * hf + e);
          float x0, x1;
          asm("{\n .reg .b64 a, b, c, d;\n"
              " mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %4};\n mov.b64 c, {%5, %6};\n"
              " fma.rn.f32x2 d, a, b, c;\n mov.b64 {%0, %1}, d;\n}\n"
              : "=f"(x0), "=f"(x1)
              : "r"(sv[e]), "r"(sv[e + 1]), "f"(sl2), "f"(nl.x), "f"(nl.y));
          const float p0 = ex2(x0), p1 = ex2(x1);
          float d0, d1;
          asm("{\n .reg .b64 a, b, c, d;\n"
              " mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n add.rn.f32x2 c, a, b;\n"
              " mov.b64 d, {%6, %7};\n mul.rn.f32x2 c, c, d;\n mov.b64 {%0, %1}, c;\n}\n"
              : "=f"(d0), "=f"(d1)
              : "r"(pv[e]), "r"(pv[e + 1]), "f"(nd.x), "f"(nd.y), "f"(p0), "f"(p1));
          pk[e >> 1] = pack_bf16(p0, p1);
          dk[e >> 1] = pack_bf16(d0, d1);
        }
        // P^T and dS^T are free once dV and dK of the previous tile have completed
        if (hf == 0 && j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.dq_done(), (j - 1) & 1, t.err));
          if (!ok) break;
        }
        tmem_st32(tPT + 32 * hf, pk);
        tmem_st32(tDS + 32 * hf, dk);
      }
      if (!ok) break;
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(bars.ds_full());
    }
    if (ok && ntile > 0) ok = mbar_wait(bars.dq_done(), (ntile - 1) & 1, t.err);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok && ntile > 0) {
      const bool wr = key < nk;
      const long long off = h * a.dkv_hs[seg] + static_cast<long long>(wr ? key : 0) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        float* out = (which ? a.dk[seg] : a.dv[seg]) + off;
        const float sc = which ? a.scale : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[32];
          tmem_ld32((which ? tK : tV) + 32 * c, w);       // warp-collective: every lane loads
          tmem_wait_ld();
          if (wr) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v = make_float4(__uint_as_float(w[e]) * sc, __uint_as_float(w[e + 1]) * sc,
                                     __uint_as_float(w[e + 2]) * sc, __uint_as_float(w[e + 3]) * sc);
              float4* p = reinterpret_cast<float4*>(out + 32 * c + e);
              if (a.dkv_accum) {
                const float4 o = *p;
                v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
              }
              *p = v;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc<TMEM_COLS>(tmem);
}

template <bool SPLIT>
cudaError_t launch_dkv_tc(const BwdTc& t, const CUtensorMap* maps, int seg, cudaStream_t st) {
  const int sm = DkvLay<SPLIT>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  dim3 grid((t.b.n_k[seg] + TBM - 1) / TBM, t.b.H);
  attn_bwd_dkv_tc_kernel<SPLIT><<<grid, BW_NTHREADS, sm, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                                                               t, seg);
  return cudaGetLastError();
}

}  // namespace

int attn_tc_tiles(long long n) { return static_cast<int>((n + TBN - 1) / TBN); }

void attn_tc_split(int H, long long n_q, int tiles_total, int* tiles_per_split, int* n_split) {
  // One CTA per SM (TMEM and shared memory), 2 x 128 query rows per CTA.  Take
  // the fewest key splits that give at least four waves over the 148 SMs, or
  // more (up to 4x) when that leaves a smaller idle tail in the last wave;
  // each split keeps at least 16 key tiles.
  constexpr long long SMS = 148;
  const long long ctas = static_cast<long long>(H) * ((n_q + 2 * TBM - 1) / (2 * TBM));
  long long maxs = tiles_total / 16;
  if (maxs < 1) maxs = 1;
  if (maxs > 4096) maxs = 4096;
  long long lo = ctas > 0 ? (4 * SMS + ctas - 1) / ctas : 1;
  if (lo < 1) lo = 1;
  if (lo > maxs) lo = maxs;
  long long best = lo;
  double best_eff = 0.0;
  for (long long ns = lo; ns <= maxs && ns <= 4 * lo; ++ns) {
    const long long tot = ctas * ns;
    const double eff = static_cast<double>(tot) / static_cast<double>(SMS * ((tot + SMS - 1) / SMS));
    if (eff > best_eff + 0.01) {
      best_eff = eff;
      best = ns;
    }
  }
  const int tps = static_cast<int>((tiles_total + best - 1) / best);
  *tiles_per_split = tps;
  *n_split = (tiles_total + tps - 1) / tps;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st) {
  CUtensorMap maps[7];
  memset(maps, 0, sizeof(maps));
  const long long H = a.H;
  if (!make_map(&maps[0], a.q, H * a.n_q)) return cudaErrorInvalidValue;
  maps[1] = maps[0];
  if (a.kc > 0 && !make_map(&maps[1], a.q_lo, H * a.n_q)) return cudaErrorInvalidValue;
  if (a.guide_only && (a.kc == 0 || a.nseg != 1 || a.n_split != 1)) return cudaErrorInvalidValue;
  if (!make_map(&maps[2], a.k[0], H * a.n_k[0])) return cudaErrorInvalidValue;
  maps[3] = maps[2];                       // guide only: V is never loaded
  if (!a.guide_only && !make_map(&maps[3], a.v[0], H * a.n_k[0])) return cudaErrorInvalidValue;
  maps[4] = maps[2];
  maps[5] = maps[3];
  if (a.nseg > 1 && (!make_map(&maps[4], a.k[1], H * a.n_k[1]) || !make_map(&maps[5], a.v[1], H * a.n_k[1])))
    return cudaErrorInvalidValue;
  maps[6] = maps[2];
  if (a.kc > 0 && !make_map(&maps[6], a.k_lo, H * a.n_k[0])) return cudaErrorInvalidValue;
  if (a.kc == 0) return launch_kc<0, false>(a, maps, st);
  if (a.excl_s) return (a.guide_only && a.kc <= 32) ? launch_kc<32, true, 2>(a, maps, st) : cudaErrorInvalidValue;
  if (a.last_s) {
    // the first of several passes (32 regions)
    if (a.kc != 32) return cudaErrorInvalidValue;
    return a.guide_only ? launch_kc<32, true, 1>(a, maps, st) : launch_kc<32, false, 1>(a, maps, st);
  }
  if (a.kc <= 8) return launch_kc2<8>(a, maps, st);
  if (a.kc <= 16) return launch_kc2<16>(a, maps, st);
  if (a.kc <= 32) return launch_kc2<32>(a, maps, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_dq_tc(const BwdArgs& b, int* err, cudaStream_t st) {
  const long long H = b.H;
  // the tensor maps address rows as head * rows + row: heads must be packed
  if (b.q_hs != static_cast<long long>(b.n_q) * D || b.do_hs != b.q_hs) return cudaErrorInvalidValue;
  for (int s = 0; s < b.nseg; ++s)
    if (b.kv_hs[s] != static_cast<long long>(b.n_k[s]) * D) return cudaErrorInvalidValue;
  const bool split = b.q_lo != nullptr;
  if (split && (b.k_lo == nullptr || b.nseg != 1)) return cudaErrorInvalidValue;
  CUtensorMap maps[8];
  memset(maps, 0, sizeof(maps));
  if (!make_map(&maps[0], b.q, H * b.n_q) || !make_map(&maps[2], b.dO, H * b.n_q)) return cudaErrorInvalidValue;
  maps[1] = maps[0];
  if (split && !make_map(&maps[1], b.q_lo, H * b.n_q)) return cudaErrorInvalidValue;
  if (!make_map(&maps[3], b.k[0], H * b.n_k[0]) || !make_map(&maps[4], b.v[0], H * b.n_k[0]))
    return cudaErrorInvalidValue;
  maps[5] = maps[3];
  maps[6] = maps[4];
  if (b.nseg > 1 && (!make_map(&maps[5], b.k[1], H * b.n_k[1]) || !make_map(&maps[6], b.v[1], H * b.n_k[1])))
    return cudaErrorInvalidValue;
  maps[7] = maps[3];
  if (split && !make_map(&maps[7], b.k_lo, H * b.n_k[0])) return cudaErrorInvalidValue;
  BwdTc t;
  t.b = b;
  t.tiles0 = attn_tc_tiles(b.n_k[0]);
  t.tiles_total = t.tiles0 + (b.nseg > 1 ? attn_tc_tiles(b.n_k[1]) : 0);
  t.err = err;
  // key-range splits fill the last wave (128-row CTAs: the split rule's row count doubles);
  // the splits add into a zeroed dq, so packed heads and an overwriting call only
  attn_tc_split(b.H, 2LL * b.n_q, t.tiles_total, &t.tiles_per_split, &t.n_split);
  if (b.dq_accum || b.dq_hs != static_cast<long long>(b.n_q) * D) {
    t.tiles_per_split = t.tiles_total;
    t.n_split = 1;
  }
  if (t.n_split > 1 && cudaMemsetAsync(b.dq, 0, static_cast<size_t>(H) * b.n_q * D * sizeof(float), st) != cudaSuccess)
    return cudaErrorUnknown;
  return split ? launch_dq_tc<true>(t, maps, st) : launch_dq_tc<false>(t, maps, st);
}

cudaError_t launch_attn_bwd_dkv_tc(const BwdArgs& b, int* err, cudaStream_t st) {
  const long long H = b.H;
  if (b.q_hs != static_cast<long long>(b.n_q) * D || b.do_hs != b.q_hs) return cudaErrorInvalidValue;
  for (int s = 0; s < b.nseg; ++s)
    if (b.kv_hs[s] != static_cast<long long>(b.n_k[s]) * D) return cudaErrorInvalidValue;
  const bool split = b.q_lo != nullptr;
  if (split && (b.k_lo == nullptr || b.nseg != 1)) return cudaErrorInvalidValue;
  CUtensorMap maps[6];
  memset(maps, 0, sizeof(maps));
  if (!make_map(&maps[0], b.q, H * b.n_q) || !make_map(&maps[2], b.dO, H * b.n_q)) return cudaErrorInvalidValue;
  maps[1] = maps[0];
  if (split && !make_map(&maps[1], b.q_lo, H * b.n_q)) return cudaErrorInvalidValue;
  BwdTc t;
  t.b = b;
  t.tiles0 = 0;
  t.tiles_total = 0;
  t.tiles_per_split = 0;
  t.n_split = 1;
  t.err = err;
  for (int seg = 0; seg < b.nseg; ++seg) {
    if (!b.dk[seg]) continue;
    if (!make_map(&maps[3], b.k[seg], H * b.n_k[seg]) || !make_map(&maps[4], b.v[seg], H * b.n_k[seg]))
      return cudaErrorInvalidValue;
    maps[5] = maps[3];
    if (split && !make_map(&maps[5], b.k_lo, H * b.n_k[0])) return cudaErrorInvalidValue;
    const cudaError_t e = split ? launch_dkv_tc<true>(t, maps, seg, st) : launch_dkv_tc<false>(t, maps, seg, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gsa
