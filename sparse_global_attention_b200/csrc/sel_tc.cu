// K3 + K4 on 5th-generation tensor cores: selection attention with the
// upsample/gate/blend fused in, for 4 x 4 compression windows (s = 4).
//
// "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (Paper-Notes, CVPR
// 2026), selection branch: each compressed query row picks its top-k regions,
// and all queries of that compression window attend to the full-resolution
// tokens of those regions ("同一压缩窗口内的 query 共享同一组 KV pair");
// gated aggregation: O_img = g * Upsample(O'_comp) + (1 - g) * O_sel with
// g = sigmoid(W_g q).
//
// A window has only s*s = 16 queries, too few for a tcgen05 MMA (M >= 64), so
// eight neighbouring windows form a group whose 128 queries fill one M = 128
// tile.  The group attends to the union of its windows' regions (about 83 of
// the 256 selections are distinct at top-32, 2.6x the per-window work),
// masked per window:
//   sel_union_kernel  one warp per group: sorts the group's (region, window) pairs and writes each
//                     distinct region once with the bit set of windows that
//                     chose it and the validity bits of its 16 tokens (pads);
//   sel_tc_kernel     persistent, two CTAs per SM, each looping over groups.
//                     TMA gathers each union region as one 4-D box
//                     [4 rows][4 cols][64] of K and of V (no multicast; pad
//                     rows/cols outside the valid grid arrive as zeros), eight
//                     regions per 128-key tile, into separate K and V rings (a
//                     K tile is free once S = Q K^T has run, a V tile only after
//                     O += P V, so K runs further ahead); the producer moves on
//                     to the next group's union entries, Q and tiles while the
//                     current group is computed.  S (SS form) and O += P V (TS
//                     form, P from TMEM) run on tcgen05 with TMEM accumulators;
//                     the softmax masks each row to its own window's regions and
//                     skips the exponentials of regions that neither window of a
//                     warp chose; G = Q W_g^T runs on the tensor core after the
//                     last S (W_g arrives as one more K tile), and the epilogue
//                     forms g, merges the VGGT fixed context (computed apart, by
//                     log-sum-exp) and writes O_img.
// Warp roles: warps 0-3 softmax and epilogue (thread = query row = TMEM lane),
// warp 4 TMA producer, warp 5 MMA issuer.  TMEM, 256 columns per CTA: S
// [0,128), O [128,192), P [192,256) bf16 pairs; G reuses S's first 64.
// All mbarrier waits are bounded (GSA_ERR_DEVICE_TIMEOUT, then drain and exit).
#include <cuda.h>

#include <vector>

#include "gsa_kernels.h"
#include "tc_ptx.cuh"

namespace gsa {

namespace {

using namespace tc;

constexpr int GW = SEL_GROUP;            // windows per group
constexpr int BOX = 16 * 128;            // one region (16 tokens) of one tensor: 2 KB
constexpr int TILE = 128 * 128;          // 128 rows of 64 bf16
constexpr int WG_BYTES = 64 * 128;       // W_g of one head
constexpr int NV = 2;                    // V ring depth
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 256;
constexpr float RESCALE_LOG2 = 8.f;      // move the reference max when it grows by > 2^8
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 64, true);
constexpr uint32_t IDESC_G = idesc_bf16(128, 64, false);

// shared memory (offsets from the 1024-byte aligned base): Q, K ring (NK), V
// ring (NV), two buffers of union entries, two of the windows' O'_comp rows, barriers
template <int NK>
struct SLay {
  static constexpr int Q = 0;
  static constexpr int K = TILE;
  static constexpr int V = K + NK * TILE;
  static constexpr int ENTS = V + NV * TILE;
  // q_full, q_free, ents_full[2], ents_free[2], k_full[NK], k_empty[NK], v_full[NV],
  // v_empty[NV], s_full, s_free, p_full, pv_done, g_full, o_read, fin
  static constexpr int NBAR = 6 + 2 * NK + 2 * NV + 7;
  static constexpr int OC_BYTES = GW * D * 4 + GW * 8;  // O'_comp rows of a group's windows (fp32),
                                                       // then per window its first token and extent
  __host__ __device__ static constexpr int ents_bytes(int emax) { return ((emax * 8 + 127) / 128) * 128; }
  __host__ __device__ static constexpr int oc(int emax) { return ENTS + 2 * ents_bytes(emax); }
  __host__ __device__ static constexpr int bar(int emax) { return oc(emax) + 2 * OC_BYTES; }
  __host__ __device__ static constexpr int bytes(int emax) { return bar(emax) + NBAR * 8 + 16 + 1024; }
};

template <int NK>
struct Bars {
  uint32_t base;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t q_free() const { return base + 8; }
  __device__ uint32_t ents_full(int b) const { return base + 8 * (2 + b); }
  __device__ uint32_t ents_free(int b) const { return base + 8 * (4 + b); }
  __device__ uint32_t k_full(int s) const { return base + 8 * (6 + s); }
  __device__ uint32_t k_empty(int s) const { return base + 8 * (6 + NK + s); }
  __device__ uint32_t v_full(int s) const { return base + 8 * (6 + 2 * NK + s); }
  __device__ uint32_t v_empty(int s) const { return base + 8 * (6 + 2 * NK + NV + s); }
  static constexpr int X = 6 + 2 * NK + 2 * NV;
  __device__ uint32_t s_full() const { return base + 8 * X; }
  __device__ uint32_t s_free() const { return base + 8 * (X + 1); }
  __device__ uint32_t p_full() const { return base + 8 * (X + 2); }
  __device__ uint32_t pv_done() const { return base + 8 * (X + 3); }
  __device__ uint32_t g_full() const { return base + 8 * (X + 4); }
  __device__ uint32_t o_read() const { return base + 8 * (X + 5); }
  __device__ uint32_t fin() const { return base + 8 * (X + 6); }
};

// the group at schedule position gs: heads in order, each head's groups in the
// order of grp_of
__device__ __forceinline__ int sched_group(const SelTcArgs& a, int gs) {
  const int h = gs / a.NG;
  return h * a.NG + __ldg(a.grp_of + (gs - h * a.NG));
}

__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// 4-D tile load (no multicast): box [1][4][4][64] of bf16 rows
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// untiled bulk copy global -> shared (no multicast), completion counted on `bar`
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// region -> (frame, region row, region col)
__device__ __forceinline__ void region_pos(int reg, int rpf, int rx, int& f, int& i, int& j) {
  f = reg / rpf;
  const int rr = reg - f * rpf;
  i = rr / rx;
  j = rr - i * rx;
}

// two exponentials with packed fp32x2 arithmetic: x = s * sl2 - mb for both,
// p = 2^x, running sums l0/l1 += p
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

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max of 16 consecutive scores (two independent chains of three-input maxima)
__device__ __forceinline__ float max16(const uint32_t* v) {
  float a = max3f(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
  float b = max3f(__uint_as_float(v[8]), __uint_as_float(v[9]), __uint_as_float(v[10]));
  a = max3f(a, __uint_as_float(v[3]), __uint_as_float(v[4]));
  b = max3f(b, __uint_as_float(v[11]), __uint_as_float(v[12]));
  a = max3f(a, __uint_as_float(v[5]), __uint_as_float(v[6]));
  b = max3f(b, __uint_as_float(v[13]), __uint_as_float(v[14]));
  return max3f(a, b, fmaxf(__uint_as_float(v[7]), __uint_as_float(v[15])));
}

// sigmoid through the hardware tanh: sigma(x) = 1/2 + tanh(x/2)/2
__device__ __forceinline__ float sigmoid_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;\n" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

// ---------------------------------------------------------------------------
// union of a group's selections
// ---------------------------------------------------------------------------
// One warp per group, eight groups per CTA: the group's pairs sorted in the
// warp's own shared-memory row, so every step synchronises a warp, not the CTA.
constexpr int UNION_WARPS = 8;

__global__ void __launch_bounds__(32 * UNION_WARPS) sel_union_kernel(const SelTcArgs a) {
  __shared__ uint32_t keys[UNION_WARPS][SEL_UNION_MAX];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = blockIdx.x * UNION_WARPS + warp, h = blockIdx.y;
  if (grp >= a.NG) return;                         // no CTA-wide barrier follows
  uint32_t* key = keys[warp];
  const int p0 = grp * GW;
  const int nw = min(GW, a.R - p0);
  const int k = a.topk;
  const int n = nw * k;
  int np2 = 2;
  while (np2 < n) np2 <<= 1;
  for (int e = lane; e < np2; e += 32) {
    uint32_t v = 0xffffffffu;
    if (e < n) {
      const int w = e / k, j = e - w * k;
      int reg = a.idx[(static_cast<long long>(h) * a.R + a.win_of[p0 + w]) * k + j];
      if (reg < 0 || reg >= a.R) {
        set_error(a.err, ERR_BOUNDS);
        reg = 0;
      }
      v = (static_cast<uint32_t>(reg) << 3) | static_cast<uint32_t>(w);
    }
    key[e] = v;
  }
  __syncwarp();
  // bitonic sort, ascending: (region, window) pairs of one region end up adjacent
  for (int size = 2; size <= np2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (np2 >> 1); i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint32_t x = key[lo], y = key[hi];
        if ((x > y) == up) {
          key[lo] = y;
          key[hi] = x;
        }
      }
      __syncwarp();
    }
  }
  // each lane takes a contiguous run of positions; the first pair of every
  // region becomes one union entry
  const int per = (np2 + 31) / 32;
  const int e0 = min(lane * per, np2), e1 = min(e0 + per, np2);
  auto first = [&](int e) {
    return key[e] != 0xffffffffu && (e == 0 || (key[e] >> 3) != (key[e - 1] >> 3));
  };
  int cnt = 0;
  for (int e = e0; e < e1; ++e) cnt += first(e) ? 1 : 0;
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += y;
  }
  int off = incl - cnt;
  uint2* out = a.uni + (static_cast<long long>(h) * a.NG + grp) * a.emax;
  for (int e = e0; e < e1; ++e) {
    if (!first(e)) continue;
    const uint32_t reg = key[e] >> 3;
    uint32_t wm = 0;
    for (int q = e; q < np2 && key[q] != 0xffffffffu && (key[q] >> 3) == reg; ++q) wm |= 1u << (key[q] & 7u);
    int f, i, j;
    region_pos(static_cast<int>(reg), a.rpf, a.rx, f, i, j);
    const int ly = min(a.g.Hv - 4 * i, 4), lx = min(a.g.Wv - 4 * j, 4);
    uint32_t kv = 0;
    for (int dy = 0; dy < ly; ++dy) kv |= ((1u << lx) - 1u) << (4 * dy);
    out[off++] = make_uint2(reg, (kv << 16) | wm);
  }
  // the last lane's end position is the number of distinct regions
  if (lane == 31) a.ucnt[static_cast<long long>(h) * a.NG + grp] = off;
}

// ---------------------------------------------------------------------------
// selection attention + gate + blend: persistent over the groups of all heads
// ---------------------------------------------------------------------------
template <int NK>
__global__ void __launch_bounds__(NTHREADS, 2)
    sel_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                  const SelTcArgs a) {
  using L = SLay<NK>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const int eb_bytes = L::ents_bytes(a.emax);
  uint2* ents0 = reinterpret_cast<uint2*>(sgen + L::ENTS);
  const Bars<NK> bars{sbase + static_cast<uint32_t>(L::bar(a.emax))};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + L::bar(a.emax) + L::NBAR * 8);

  const int warp = threadIdx.x >> 5;
  const int total = a.H * a.NG;                        // groups of all heads (< 2^31, checked at launch)
  const bool learned = a.gate_mode == 0;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.q_free(), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars.ents_full(b), 32);
      mbar_init(bars.ents_free(b), 4);
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.s_free(), 4);
    mbar_init(bars.p_full(), 4);
    mbar_init(bars.pv_done(), 1);
    mbar_init(bars.g_full(), 1);
    mbar_init(bars.o_read(), 4);
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
    const int lane = threadIdx.x & 31;
    bool ok = true;
    int kq = 0, vq = 0;                                // K / V tiles issued (ring positions)
    int nq = 0;                                        // Q tiles issued
    int n = 0;
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    for (int gs = blockIdx.x; ok && gs < total; gs += gridDim.x, ++n) {
      const int gi = sched_group(a, gs);
      const int h = gi / a.NG;
      const int p0 = (gi - h * a.NG) * GW;
      const int fh = h * a.F;                          // first frame of this head in the 4-D maps
      const int eb = n & 1;
      uint2* ents = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(ents0) + eb * eb_bytes);
      // this buffer (entries, O'_comp rows) held group n - 2's until its epilogue was done
      if (n >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bars.ents_free(eb), ((n - 2) >> 1) & 1, a.err));
        if (!ok) break;
      }
      const int nu = min(a.ucnt[gi], a.emax);
      const int nt = (nu + 7) >> 3;
      const uint2* src = a.uni + static_cast<long long>(gi) * a.emax;
      for (int u = lane; u < nu; u += 32) ents[u] = src[u];
      // the group's windows: region, and for the epilogue its first token and valid extent
      const int nwin = min(GW, a.R - p0);
      int wr = 0, wf = 0, wi = 0, wj = 0;
      if (lane < nwin) {
        wr = a.win_of[p0 + lane];
        region_pos(wr, a.rpf, a.rx, wf, wi, wj);
      }
      if (lane < GW) {
        int2* wd = reinterpret_cast<int2*>(sgen + L::oc(a.emax) + eb * L::OC_BYTES + GW * D * 4);
        const int ly = lane < nwin ? min(a.g.Hv - 4 * wi, 4) : 0, lx = lane < nwin ? min(a.g.Wv - 4 * wj, 4) : 0;
        wd[lane] = make_int2((wf * a.g.Hp + 4 * wi) * a.g.Wp + 4 * wj, (ly << 8) | lx);
      }
      mbar_arrive(bars.ents_full(eb));                  // every lane: its entries and windows are written
      __syncwarp();
      // Q of this group once the previous group's last MMA that reads Q has completed
      if (n >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(bars.q_free(), (n - 1) & 1, a.err));
        if (!ok) break;
      }
      // Q (8 window boxes) and, unless g = 0, the windows' O'_comp rows
      const bool need_oc = a.gate_mode != 2;
      if (lane == 0) mbar_expect_tx(bars.q_full(), TILE + (need_oc ? nwin * D * 4 : 0));
      __syncwarp();
      if (lane < GW) {
        // rows past the grid: zeros
        tma_load_4d(sbase + L::Q + lane * BOX, &tm_q, 0, 4 * wj, lane < nwin ? 4 * wi : a.g.Hv, fh + wf, bars.q_full());
        if (need_oc && lane < nwin)
          bulk_load(sbase + L::oc(a.emax) + eb * L::OC_BYTES + lane * D * 4,
                    a.o_comp + (static_cast<long long>(h) * a.R + wr) * D, D * 4, bars.q_full());
      }
      ++nq;
      // step u: K tile u (u = nt: W_g) and V tile u - 1; K runs a tile ahead of V
      const int nk_tiles = nt + (learned ? 1 : 0);
      for (int u = 0; u <= nt; ++u) {
        if (u < nk_tiles) {
          const int s = static_cast<int>(kq % NK);
          if (kq >= NK && !__all_sync(0xffffffffu, mbar_wait(bars.k_empty(s), ((kq / NK) - 1) & 1, a.err))) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + L::K + s * TILE;
          if (u < nt) {
            if (lane == 0) mbar_expect_tx(bars.k_full(s), TILE);
            __syncwarp();
            if (lane < 8) {
              const int e = 8 * u + lane;
              int f = 0, i = 0, j = 0, y = a.g.Hv;      // past the union: zeros
              if (e < nu) {
                region_pos(static_cast<int>(ents[e].x), a.rpf, a.rx, f, i, j);
                y = 4 * i;
              }
              tma_load_4d(dst + lane * BOX, &tm_k, 0, 4 * j, y, fh + f, bars.k_full(s));
            }
          } else if (lane == 0) {
            mbar_expect_tx(bars.k_full(s), WG_BYTES);
            tma_load_2d(dst, &tm_w, 0, h * 64, bars.k_full(s));
          }
          __syncwarp();
          ++kq;
        }
        if (u >= 1) {
          const int t = u - 1;
          const int s = static_cast<int>(vq % NV);
          if (vq >= NV && !__all_sync(0xffffffffu, mbar_wait(bars.v_empty(s), ((vq / NV) - 1) & 1, a.err))) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_expect_tx(bars.v_full(s), TILE);
          __syncwarp();
          if (lane < 8) {
            const int e = 8 * t + lane;
            int f = 0, i = 0, j = 0, y = a.g.Hv;
            if (e < nu) {
              region_pos(static_cast<int>(ents[e].x), a.rpf, a.rx, f, i, j);
              y = 4 * i;
            }
            tma_load_4d(sbase + L::V + s * TILE + lane * BOX, &tm_v, 0, 4 * j, y, fh + f, bars.v_full(s));
          }
          __syncwarp();
          ++vq;
        }
      }
    }
    // drain: every issued copy has landed before the CTA may exit
    for (int q = kq > NK ? kq - NK : 0; q < kq; ++q) mbar_wait(bars.k_full(q % NK), (q / NK) & 1, a.err);
    for (int q = vq > NV ? vq - NV : 0; q < vq; ++q) mbar_wait(bars.v_full(q % NV), (q / NV) & 1, a.err);
    if (nq > 0) mbar_wait(bars.q_full(), (nq - 1) & 1, a.err);
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    const uint64_t dq = sdesc_sw128(sbase + L::Q, 16, 1024);
    const uint64_t dk0 = sdesc_sw128(sbase + L::K, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(sbase + L::V, 8192, 1024);
    constexpr uint32_t T16 = TILE >> 4;
    bool ok = true;
    int kq = 0, vq = 0;                                // K / V tiles consumed
    int T = 0;                                         // tiles of all groups so far
    int n = 0;
    for (int gs = blockIdx.x; ok && gs < total; gs += gridDim.x, ++n) {
      const int gi = sched_group(a, gs);
      const int nu = min(a.ucnt[gi], a.emax);
      const int nt = (nu + 7) >> 3;
      ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), n & 1, a.err));
      if (!ok) break;
      // S and O of the previous group have been read by its epilogue
      if (n >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(bars.o_read(), (n - 1) & 1, a.err));
        if (!ok) break;
      }
      tc_fence_after();
      for (int j = 0; j <= nt; ++j) {
        if (j < nt) {
          const int s = static_cast<int>(kq % NK);
          ok = __all_sync(0xffffffffu, mbar_wait(bars.k_full(s), (kq / NK) & 1, a.err));
          if (!ok) break;
          if (j > 0) {
            // S_j overwrites S_{j-1}: the softmax warps have read it
            ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (T + j - 1) & 1, a.err));
            if (!ok) break;
          }
          tc_fence_after();
          if (leader) {
            const uint64_t dk = dk0 + s * T16;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem, dq + 2 * ks, dk + 2 * ks, IDESC_S, ks > 0 ? 1u : 0u);
            mma_commit(bars.s_full());
            mma_commit(bars.k_empty(s));
          }
          __syncwarp();
          ++kq;
        }
        if (j > 0) {
          // O += P_{j-1} V_{j-1}: P from TMEM (TS form), V MN-major in shared memory
          const int s = static_cast<int>(vq % NV);
          ok = __all_sync(0xffffffffu, mbar_wait(bars.v_full(s), (vq / NV) & 1, a.err));
          if (!ok) break;
          ok = __all_sync(0xffffffffu, mbar_wait(bars.p_full(), (T + j - 1) & 1, a.err));
          if (!ok) break;
          tc_fence_after();
          if (leader) {
            const uint64_t dv = dv0 + s * T16;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_bf16_ts(tmem + 128, tmem + 192 + 8 * ks, dv + ks * 128, IDESC_PV, (j > 1 || ks > 0) ? 1u : 0u);
            mma_commit(bars.pv_done());
            mma_commit(bars.v_empty(s));
          }
          __syncwarp();
          ++vq;
        }
      }
      if (!ok) break;
      if (learned) {
        // G = Q W_g^T into S's first 64 columns once the last S has been read; W_g is
        // the next K tile
        const int s = static_cast<int>(kq % NK);
        ok = __all_sync(0xffffffffu, mbar_wait(bars.k_full(s), (kq / NK) & 1, a.err));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (T + nt - 1) & 1, a.err));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint64_t dw = dk0 + s * T16;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem, dq + 2 * ks, dw + 2 * ks, IDESC_G, ks > 0 ? 1u : 0u);
          mma_commit(bars.g_full());
          mma_commit(bars.k_empty(s));
        }
        __syncwarp();
        ++kq;
      }
      // every MMA that reads this group's Q has been issued
      if (leader) mma_commit(bars.q_free());
      __syncwarp();
      T += nt;
    }
    if (leader) mma_commit(bars.fin());
    __syncwarp();
    mbar_wait(bars.fin(), 0, a.err);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x;                         // query row of the group = TMEM lane
    const int w = r >> 4;                              // its window in the group
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off, tO = tS + 128, tP = tS + 192;
    const float sl2 = a.scale_log2;
    const uint32_t wsh = 2u * warp;                    // the warp's two windows: bits wsh, wsh + 1
    const long long img_hs = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
    const float gfix = a.gate_mode == 1 ? 1.f : 0.f;
    bool ok = true;
    int T = 0;                                         // tiles of all groups so far
    int n = 0;
    for (int gs = blockIdx.x; ok && gs < total; gs += gridDim.x, ++n) {
      const int gi = sched_group(a, gs);
      const int h = gi / a.NG;
      const int p0 = (gi - h * a.NG) * GW;
      const int eb = n & 1;
      const uint2* ents = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(ents0) + eb * eb_bytes);
      const int nu = min(a.ucnt[gi], a.emax);
      const int nt = (nu + 7) >> 3;
      ok = __all_sync(0xffffffffu, mbar_wait(bars.ents_full(eb), (n >> 1) & 1, a.err));
      // the group's Q and O'_comp rows have landed (read in the epilogue); Q of the
      // next group cannot arrive before this group's MMAs are done, so the phase
      // waited for here is this group's
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), n & 1, a.err));
      float m = -INFINITY, l = 0.f;
      for (int t = 0; ok && t < nt; ++t) {
        const int Tt = T + t;
        // the tile's eight regions, read while S is computed: bit e = one of the warp's
        // windows chose region e, bit 8 + e = this row's window chose it, bit 16 + e =
        // region e has tokens outside the valid grid
        uint32_t tb = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int u = 8 * t + e;
          const uint32_t y = u < nu ? ents[u].y : 0xffff0000u;
          tb |= ((((y >> wsh) & 3u) != 0u ? 1u : 0u) << e) | (((y >> w) & 1u) << (8 + e)) |
                ((y >> 16) != 0xffffu ? 1u << (16 + e) : 0u);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full(), Tt & 1, a.err));
        if (!ok) break;
        tc_fence_after();
        float l0 = 0.f, l1 = 0.f;
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t v[64];
          tmem_ld64(tS + 64 * hf, v);
          const uint32_t act = (tb >> (4 * hf)) & 15u, rsel = (tb >> (8 + 4 * hf)) & 15u;
          tmem_wait_ld();
          if (hf == 1) {
            tc_fence_before();
            warp_arrive(bars.s_free());
          }
          // a row takes a region only if its own window chose it: that enters the max
          // as one select per region and the exponentials as an infinite offset; chosen
          // regions with pad tokens (warp-uniform) mask those tokens one by one
          const uint32_t pm = (tb >> (16 + 4 * hf)) & act;
          if (pm) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (pm & (1u << e)) {
                const uint32_t kv = ents[8 * t + 4 * hf + e].y >> 16;
#pragma unroll
                for (int c = 0; c < 16; ++c) v[16 * e + c] = ((kv >> c) & 1u) ? v[16 * e + c] : 0xff800000u;
              }
            }
          }
          float hmx = -INFINITY;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float mx = max16(v + 16 * e);
            hmx = ((rsel >> e) & 1u) ? fmaxf(hmx, mx) : hmx;
          }
          // online softmax: the reference max moves only when this half raises the
          // row's max by more than 2^8
          const bool grow = (m == -INFINITY) ? (hmx != -INFINITY) : ((hmx - m) * sl2 > RESCALE_LOG2);
          if (__any_sync(0xffffffffu, grow)) {
            l += l0 + l1;
            l0 = l1 = 0.f;
            // rows that had a finite max scale what they accumulated (their O and
            // this tile's first half of P); a row without one has only zeros there
            const bool resc = grow && m != -INFINITY;
            const float alpha = resc ? ex2((m - hmx) * sl2) : 1.f;
            if (grow) m = hmx;
            l *= alpha;
            const bool any_resc = __any_sync(0xffffffffu, resc);
            if (t > 0 && any_resc) {
              // O holds this group's earlier tiles: rescale it once the previous P V has landed
              ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(), (Tt - 1) & 1, a.err));
              if (!ok) break;
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < 8; ++c) {
                uint32_t q[8];
                tmem_ld8(tO + 8 * c, q);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) q[e] = __float_as_uint(__uint_as_float(q[e]) * alpha);
                tmem_st8(tO + 8 * c, q);
              }
            }
            if (hf == 1 && any_resc) {
              // the first half's P was written against the old max
              tmem_wait_st();
#pragma unroll 1
              for (int c = 0; c < 4; ++c) {
                uint32_t q[8];
                tmem_ld8(tP + 8 * c, q);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&q[e]);
                  q[e] = pack_bf16(__low2float(b) * alpha, __high2float(b) * alpha);
                }
                tmem_st8(tP + 8 * c, q);
              }
            }
          }
          const float mb = (m == -INFINITY) ? 0.f : m * sl2;
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (act & (1u << e)) {
              const float nmb = ((rsel >> e) & 1u) ? -mb : -INFINITY;
#pragma unroll
              for (int c = 0; c < 16; c += 2) {
                float p0, p1;
                exp2_pair(v[16 * e + c], v[16 * e + c + 1], sl2, nmb, l0, l1, p0, p1);
                pk[8 * e + (c >> 1)] = pack_bf16(p0, p1);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 8; ++c) pk[8 * e + c] = 0u;
            }
          }
          // P is free once the previous tile's P V (of this or the previous group) has
          // completed: waited for only now, so that P V overlaps the exponentials
          if (hf == 0 && Tt > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(), (Tt - 1) & 1, a.err));
            if (!ok) break;
          }
          tmem_st32(tP + 32 * hf, pk);
        }
        if (!ok) break;
        l += l0 + l1;
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(bars.p_full());
      }
      T += nt;
      if (!ok) break;
      // ---- epilogue --------------------------------------------------------
      const int q = r & 15;
      const bool in_grp = p0 + w < a.R;
      const int2 wd = reinterpret_cast<const int2*>(sgen + L::oc(a.emax) + eb * L::OC_BYTES + GW * D * 4)[w];
      const int dy = q >> 2, dx = q & 3;
      const bool qv = in_grp && dy < (wd.y >> 8) && dx < (wd.y & 0xff);
      const long long tok = static_cast<long long>(wd.x) + dy * a.g.Wp + dx;
      const long long ft = static_cast<long long>(h) * img_hs + tok;
      const float lf = (a.fix_o && qv) ? a.fix_lse[ft] : -INFINITY;
      ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(), (T - 1) & 1, a.err));
      if (ok && learned) ok = __all_sync(0xffffffffu, mbar_wait(bars.g_full(), n & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      // merge with the fixed context's attention (normalised O_fix, base-2 LSE L_fix):
      // O = (O_fix 2^(L_fix - M) + o 2^(m sl2 - M)) / (2^(L_fix - M) + l 2^(m sl2 - M))
      float inv = (qv && l > 0.f) ? 1.f / l : 0.f, wfix = 0.f;
      const float* fo = nullptr;
      if (a.fix_o && qv) {
        const float md = l > 0.f ? m * sl2 : -INFINITY;
        const float mm = fmaxf(lf, md);
        const float wf = ex2(lf - mm), wd = l > 0.f ? ex2(md - mm) : 0.f;
        const float den = wf + l * wd;
        inv = den > 0.f ? wd / den : 0.f;
        wfix = den > 0.f ? wf / den : 0.f;
        fo = a.fix_o + ft * D;
      }
      const float* ocs = reinterpret_cast<const float*>(sgen + L::oc(a.emax) + eb * L::OC_BYTES) + w * D;
      __nv_bfloat16* oi = a.o_img + static_cast<long long>(h) * img_hs * D + tok * D;
      __nv_bfloat16* os = a.o_sel ? a.o_sel + static_cast<long long>(h) * img_hs * D + tok * D : nullptr;
      // O and G in two halves; once the second is in registers the next group's S
      // and P V may overwrite TMEM
#pragma unroll 1
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t ov[32], gv[32];
        tmem_ld32(tO + c0, ov);
        if (learned) tmem_ld32(tS + c0, gv);
        tmem_wait_ld();
        if (c0 == 32) {
          tc_fence_before();
          warp_arrive(bars.o_read());
        }
#pragma unroll
        for (int e0 = 0; e0 < 32; e0 += 8) {
          uint32_t po[4], ps[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int c = c0 + e0 + e;
            float s0 = __uint_as_float(ov[e0 + e]) * inv, s1 = __uint_as_float(ov[e0 + e + 1]) * inv;
            if (fo) {
              const float2 of = __ldg(reinterpret_cast<const float2*>(fo + c));
              s0 = fmaf(of.x, wfix, s0);
              s1 = fmaf(of.y, wfix, s1);
            }
            float g0 = gfix, g1 = gfix;
            if (learned) {
              g0 = sigmoid_tanh(__uint_as_float(gv[e0 + e]));
              g1 = sigmoid_tanh(__uint_as_float(gv[e0 + e + 1]));
            }
            // g = 0 (selection only, or no compressed value) never reads O'_comp
            const float2 cv = (a.gate_mode == 2 || !qv) ? make_float2(0.f, 0.f)
                                                        : *reinterpret_cast<const float2*>(ocs + c);
            po[e >> 1] = pack_bf16(qv ? g0 * cv.x + (1.f - g0) * s0 : 0.f, qv ? g1 * cv.y + (1.f - g1) * s1 : 0.f);
            ps[e >> 1] = pack_bf16(qv ? s0 : 0.f, qv ? s1 : 0.f);
          }
          if (in_grp) {
            *reinterpret_cast<uint4*>(oi + c0 + e0) = make_uint4(po[0], po[1], po[2], po[3]);
            if (os) *reinterpret_cast<uint4*>(os + c0 + e0) = make_uint4(ps[0], ps[1], ps[2], ps[3]);
          }
        }
      }
      // this group's entries and O'_comp rows are no longer read
      warp_arrive(bars.ents_free(eb));
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

// image tokens [frames of all heads][Hp][Wp][64] bf16 seen as the 4-D tensor
// (64, Wv, Hv, frames) with the padded strides: a box of [4 rows][4 cols]
// reads zeros outside the valid grid
bool make_region_map(CUtensorMap* m, const void* base, const Grid& g, long long frames) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base || frames <= 0 || frames > 0x7fffffffLL) return false;
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(g.Wv), static_cast<cuuint64_t>(g.Hv),
                              static_cast<cuuint64_t>(frames)};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(g.Wp) * 128,
                                 static_cast<cuuint64_t>(g.Hp) * g.Wp * 128};
  const cuuint32_t box[4] = {64, 4, 4, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W_g of every head, [H * 64][64] bf16, 64-row boxes
bool make_wg_map(CUtensorMap* m, const void* base, int H) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !base) return false;
  const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(H) * 64};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int sel_group_count(int R) { return (R + SEL_GROUP - 1) / SEL_GROUP; }

void sel_group_order(int F, int rows, int cols, int* win_of) {
  // per frame: row pairs top to bottom, columns alternately left to right and
  // right to left, the pair's two windows of a column next to each other
  int p = 0;
  for (int f = 0; f < F; ++f)
    for (int pr = 0; 2 * pr < rows; ++pr)
      for (int cc = 0; cc < cols; ++cc) {
        const int c = (pr & 1) ? cols - 1 - cc : cc;
        for (int rr = 2 * pr; rr < 2 * pr + 2 && rr < rows; ++rr) win_of[p++] = (f * rows + rr) * cols + c;
      }
}

void sel_group_schedule(int F, int rpf, int NG, int* grp_of) {
  // key of a group: (position of its first window inside the frame, frame); a stable
  // counting sort over the positions keeps frames in order within a position
  std::vector<int> cnt(rpf + 1, 0);
  for (int g = 0; g < NG; ++g) ++cnt[(g * GW) % rpf + 1];
  for (int p = 0; p < rpf; ++p) cnt[p + 1] += cnt[p];
  for (int g = 0; g < NG; ++g) grp_of[cnt[(g * GW) % rpf]++] = g;
  (void)F;
}

cudaError_t launch_sel_union(const SelTcArgs& a, cudaStream_t st) {
  if (a.emax > SEL_UNION_MAX || a.topk * SEL_GROUP > a.emax) return cudaErrorInvalidValue;
  dim3 grid((a.NG + UNION_WARPS - 1) / UNION_WARPS, a.H);
  sel_union_kernel<<<grid, 32 * UNION_WARPS, 0, st>>>(a);
  return cudaGetLastError();
}

template <int NK>
cudaError_t launch_sel_tc_nk(const SelTcArgs& a, const CUtensorMap* maps, cudaStream_t st) {
  const int sm = SLay<NK>::bytes(a.emax);
  cudaError_t e = cudaFuncSetAttribute(sel_tc_kernel<NK>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cudaErrorInvalidValue;
  }
  const long long total = static_cast<long long>(a.H) * a.NG;
  if (total >= (1LL << 31)) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(total < 2LL * sms ? total : 2LL * sms);
  sel_tc_kernel<NK><<<grid, NTHREADS, sm, st>>>(maps[0], maps[1], maps[2], maps[3], a);
  return cudaGetLastError();
}

cudaError_t launch_sel_tc(const SelTcArgs& a, cudaStream_t st) {
  CUtensorMap maps[4];
  const long long frames = static_cast<long long>(a.H) * a.F;
  if (!make_region_map(&maps[0], a.q_img, a.g, frames) || !make_region_map(&maps[1], a.k_img, a.g, frames) ||
      !make_region_map(&maps[2], a.v_img, a.g, frames))
    return cudaErrorInvalidValue;
  if (a.gate_mode == 0) {
    if (!make_wg_map(&maps[3], a.w_g, a.H)) return cudaErrorInvalidValue;
  } else {
    maps[3] = maps[0];                                   // never read
  }
  // three K stages while two CTAs of the union lists still fit an SM, else two
  return a.emax <= 256 ? launch_sel_tc_nk<3>(a, maps, st) : launch_sel_tc_nk<2>(a, maps, st);
}

}  // namespace gsa
