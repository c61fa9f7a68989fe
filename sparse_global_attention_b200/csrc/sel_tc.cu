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
//   sel_union_kernel  sorts the group's (region, window) pairs and writes each
//                     distinct region once with the bit set of windows that
//                     chose it and the validity bits of its 16 tokens (pads);
//   sel_tc_kernel     one CTA per group: TMA gathers each union region as one
//                     4-D box [4 rows][4 cols][64] of K and of V (no multicast;
//                     pad rows/cols outside the valid grid arrive as zeros),
//                     eight regions per 128-key tile; S = Q K^T (SS form) and
//                     O += P V (TS form, P from TMEM) on tcgen05 with TMEM
//                     accumulators; the softmax masks each row to its own
//                     window's regions and skips the exponentials of regions
//                     that neither window of a warp chose; after the last tile
//                     G = Q W_g^T runs on the tensor core and the epilogue
//                     forms g, merges the VGGT fixed context (computed apart,
//                     by log-sum-exp) and writes O_img.
// Warp roles: warps 0-3 softmax (thread = query row = TMEM lane), warp 4 TMA
// producer, warp 5 MMA issuer.  Two CTAs per SM (TMEM: 256 columns each:
// S [0,128), O [128,192), P [192,256) bf16 pairs; G reuses S's first 64).
// All mbarrier waits are bounded (GSA_ERR_DEVICE_TIMEOUT, then drain and exit).
#include <cuda.h>

#include "gsa_kernels.h"
#include "tc_ptx.cuh"

namespace gsa {

namespace {

using namespace tc;

constexpr int GW = SEL_GROUP;            // windows per group
constexpr int BOX = 16 * 128;            // one region (16 tokens) of one tensor: 2 KB
constexpr int TILE = 128 * 128;          // 128 rows of 64 bf16
constexpr int WG_BYTES = 64 * 128;       // W_g of one head
constexpr int NST = 2;                   // K/V ring depth
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 256;
constexpr float RESCALE_LOG2 = 8.f;      // move the reference max when it grows by > 2^8
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 64, true);
constexpr uint32_t IDESC_G = idesc_bf16(128, 64, false);

// shared memory (offsets from the 1024-byte aligned base)
constexpr int OFF_Q = 0;
constexpr int OFF_WG = TILE;
constexpr int OFF_RING = TILE + WG_BYTES;
constexpr int STAGE = 2 * TILE;          // K tile, then V tile
constexpr int OFF_ENTS = OFF_RING + NST * STAGE;
// barriers after the union entries: q_full, ents, full[NST], empty[NST], s_full, s_free,
// p_full, pv_done, g_full, fin
constexpr int NBAR = 2 + 2 * NST + 6;

__host__ __device__ constexpr int smem_bytes(int emax) {
  return OFF_ENTS + ((emax * 8 + 127) / 128) * 128 + NBAR * 8 + 16 + 1024;
}

struct Bars {
  uint32_t base;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t ents() const { return base + 8; }
  __device__ uint32_t full(int s) const { return base + 8 * (2 + s); }
  __device__ uint32_t empty(int s) const { return base + 8 * (2 + NST + s); }
  __device__ uint32_t s_full() const { return base + 8 * (2 + 2 * NST); }
  __device__ uint32_t s_free() const { return base + 8 * (3 + 2 * NST); }
  __device__ uint32_t p_full() const { return base + 8 * (4 + 2 * NST); }
  __device__ uint32_t pv_done() const { return base + 8 * (5 + 2 * NST); }
  __device__ uint32_t g_full() const { return base + 8 * (6 + 2 * NST); }
  __device__ uint32_t fin() const { return base + 8 * (7 + 2 * NST); }
};

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

// sigmoid through the hardware tanh: sigma(x) = 1/2 + tanh(x/2)/2
__device__ __forceinline__ float sigmoid_tanh(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;\n" : "=f"(t) : "f"(0.5f * x));
  return fmaf(0.5f, t, 0.5f);
}

// ---------------------------------------------------------------------------
// union of a group's selections
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) sel_union_kernel(const SelTcArgs a) {
  __shared__ uint32_t key[SEL_UNION_MAX];
  __shared__ int wsum[8];
  const int grp = blockIdx.x, h = blockIdx.y;
  const int p0 = grp * GW;
  const int nw = min(GW, a.R - p0);
  const int k = a.topk;
  const int n = nw * k;
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int e = threadIdx.x; e < np2; e += blockDim.x) {
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
  __syncthreads();
  // bitonic sort, ascending: (region, window) pairs of one region end up adjacent
  for (int size = 2; size <= np2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (np2 >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint32_t x = key[lo], y = key[hi];
        if ((x > y) == up) {
          key[lo] = y;
          key[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  // each thread takes a contiguous run of positions; the first pair of every
  // region becomes one union entry
  const int per = (np2 + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per, e1 = min(e0 + per, np2);
  auto first = [&](int e) {
    return key[e] != 0xffffffffu && (e == 0 || (key[e] >> 3) != (key[e - 1] >> 3));
  };
  int cnt = 0;
  for (int e = e0; e < e1; ++e) cnt += first(e) ? 1 : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int off = incl - cnt;
  for (int q = 0; q < warp; ++q) off += wsum[q];
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
  // the last thread's end position is the number of distinct regions
  if (threadIdx.x == blockDim.x - 1) a.ucnt[static_cast<long long>(h) * a.NG + grp] = off;
}

// ---------------------------------------------------------------------------
// selection attention of one group + gate + blend
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NTHREADS, 2)
    sel_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                  const SelTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  uint2* ents = reinterpret_cast<uint2*>(sgen + OFF_ENTS);
  const int ents_bytes = ((a.emax * 8 + 127) / 128) * 128;
  const Bars bars{sbase + OFF_ENTS + ents_bytes};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + OFF_ENTS + ents_bytes + NBAR * 8);

  const int warp = threadIdx.x >> 5;
  const int grp = blockIdx.x, h = blockIdx.y;
  const int p0 = grp * GW;
  const long long gi = static_cast<long long>(h) * a.NG + grp;
  const int nu = min(a.ucnt[gi], a.emax);
  const int nt = (nu + 7) >> 3;                       // 128-key tiles (8 regions each)
  const bool learned = a.gate_mode == 0;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    mbar_init(bars.ents(), 32);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.s_free(), 4);
    mbar_init(bars.p_full(), 4);
    mbar_init(bars.pv_done(), 1);
    mbar_init(bars.g_full(), 1);
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
    const uint2* src = a.uni + gi * a.emax;
    for (int u = lane; u < nu; u += 32) ents[u] = src[u];
    mbar_arrive(bars.ents());                          // every lane: its entries are written
    __syncwarp();
    const bool leader = elect_one();
    const int fh = h * a.F;                            // first frame of this head in the 4-D maps
    if (leader) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_expect_tx(bars.q_full(), TILE + (learned ? WG_BYTES : 0));
      for (int w = 0; w < GW; ++w) {
        int f = 0, i = 0, j = 0, y = a.g.Hv;           // rows past the grid: zeros
        if (p0 + w < a.R) {
          region_pos(a.win_of[p0 + w], a.rpf, a.rx, f, i, j);
          y = 4 * i;
        }
        tma_load_4d(sbase + OFF_Q + w * BOX, &tm_q, 0, 4 * j, y, fh + f, bars.q_full());
      }
      if (learned) tma_load_2d(sbase + OFF_WG, &tm_w, 0, h * 64, bars.q_full());
    }
    __syncwarp();
    int issued = 0;
    for (int t = 0; t < nt; ++t) {
      const int s = t % NST;
      if (t >= NST && !__all_sync(0xffffffffu, mbar_wait(bars.empty(s), ((t / NST) - 1) & 1, a.err))) break;
      const uint32_t st = sbase + OFF_RING + s * STAGE;
      if (leader) {
        mbar_expect_tx(bars.full(s), 2 * TILE);
        for (int e = 0; e < 8; ++e) {
          const int u = 8 * t + e;
          int f = 0, i = 0, j = 0, y = a.g.Hv;         // past the union: zeros
          if (u < nu) {
            region_pos(static_cast<int>(ents[u].x), a.rpf, a.rx, f, i, j);
            y = 4 * i;
          }
          tma_load_4d(st + e * BOX, &tm_k, 0, 4 * j, y, fh + f, bars.full(s));
          tma_load_4d(st + TILE + e * BOX, &tm_v, 0, 4 * j, y, fh + f, bars.full(s));
        }
      }
      __syncwarp();
      ++issued;
    }
    // drain: every issued copy has landed before the CTA may exit
    for (int t = max(0, issued - NST); t < issued; ++t) mbar_wait(bars.full(t % NST), (t / NST) & 1, a.err);
    mbar_wait(bars.q_full(), 0, a.err);
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    constexpr uint32_t ST16 = STAGE >> 4;
    const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
    const uint64_t dw = sdesc_sw128(sbase + OFF_WG, 16, 1024);
    const uint64_t dk0 = sdesc_sw128(sbase + OFF_RING, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(sbase + OFF_RING + TILE, 8192, 1024);
    bool ok = __all_sync(0xffffffffu, mbar_wait(bars.q_full(), 0, a.err));
    tc_fence_after();
    for (int j = 0; ok && j <= nt; ++j) {
      if (j < nt) {
        ok = __all_sync(0xffffffffu, mbar_wait(bars.full(j % NST), (j / NST) & 1, a.err));
        if (!ok) break;
        if (j > 0) {
          // S_j overwrites S_{j-1}: the softmax warps have read it
          ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (j - 1) & 1, a.err));
          if (!ok) break;
        }
        tc_fence_after();
        const uint64_t dk = dk0 + (j % NST) * ST16;
        if (leader) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem, dq + 2 * ks, dk + 2 * ks, IDESC_S, ks > 0 ? 1u : 0u);
          mma_commit(bars.s_full());
        }
        __syncwarp();
      }
      if (j > 0) {
        // O += P_{j-1} V_{j-1}: P from TMEM (TS form), V MN-major in shared memory
        ok = __all_sync(0xffffffffu, mbar_wait(bars.p_full(), (j - 1) & 1, a.err));
        if (!ok) break;
        tc_fence_after();
        const uint64_t dv = dv0 + ((j - 1) % NST) * ST16;
        if (leader) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16_ts(tmem + 128, tmem + 192 + 8 * ks, dv + ks * 128, IDESC_PV, (j > 1 || ks > 0) ? 1u : 0u);
          mma_commit(bars.pv_done());
          mma_commit(bars.empty((j - 1) % NST));
        }
        __syncwarp();
      }
    }
    if (ok && learned && nt > 0) {
      // G = Q W_g^T into S's first 64 columns, once the last S has been read
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_free(), (nt - 1) & 1, a.err));
      tc_fence_after();
      if (ok && leader) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_bf16_ss(tmem, dq + 2 * ks, dw + 2 * ks, IDESC_G, ks > 0 ? 1u : 0u);
        mma_commit(bars.g_full());
      }
      __syncwarp();
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
    float m = -INFINITY, l = 0.f;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bars.ents(), 0, a.err));
    for (int t = 0; ok && t < nt; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full(), t & 1, a.err));
      if (!ok) break;
      tc_fence_after();
      float l0 = 0.f, l1 = 0.f;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t v[64];
        tmem_ld64(tS + 64 * hf, v);
        // the half's four regions: window bits and token validity
        uint32_t info[4];
        uint32_t act = 0;                              // bit e: a region one of the warp's windows chose
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int u = 8 * t + 4 * hf + e;
          info[e] = u < nu ? ents[u].y : 0u;
          act |= (((info[e] >> wsh) & 3u) != 0u ? 1u : 0u) << e;
        }
        tmem_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          warp_arrive(bars.s_free());
        }
        float hmx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (act & (1u << e)) {
            const uint32_t kv = ((info[e] >> w) & 1u) ? (info[e] >> 16) : 0u;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t x = ((kv >> c) & 1u) ? v[16 * e + c] : 0xff800000u;   // -inf
              v[16 * e + c] = x;
              hmx = fmaxf(hmx, __uint_as_float(x));
            }
          }
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
            // O holds earlier tiles: rescale it once the previous P V has landed
            ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(), (t - 1) & 1, a.err));
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
        // P is free once the previous tile's P V has completed
        if (hf == 0 && t > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done(), (t - 1) & 1, a.err));
          if (!ok) break;
        }
        const float mb = (m == -INFINITY) ? 0.f : m * sl2;
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (act & (1u << e)) {
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              float p0, p1;
              exp2_pair(v[16 * e + c], v[16 * e + c + 1], sl2, -mb, l0, l1, p0, p1);
              pk[8 * e + (c >> 1)] = pack_bf16(p0, p1);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) pk[8 * e + c] = 0u;
          }
        }
        tmem_st32(tP + 32 * hf, pk);
      }
      if (!ok) break;
      l += l0 + l1;
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(bars.p_full());
    }
    // ---- epilogue ----------------------------------------------------------
    if (ok && nt > 0) ok = mbar_wait(bars.pv_done(), (nt - 1) & 1, a.err);
    ok = __all_sync(0xffffffffu, ok);
    bool gok = ok;
    if (ok && learned) gok = __all_sync(0xffffffffu, mbar_wait(bars.g_full(), 0, a.err));
    tc_fence_after();
    const int pw = p0 + w;
    const int q = r & 15;
    int f = 0, i = 0, j = 0;
    const bool in_grp = pw < a.R;
    const int wr = in_grp ? a.win_of[pw] : 0;
    region_pos(wr, a.rpf, a.rx, f, i, j);
    const int y = 4 * i + (q >> 2), x = 4 * j + (q & 3);
    const bool qv = in_grp && y < a.g.Hv && x < a.g.Wv;
    const long long tok = (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x;
    const long long img_hs = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
    // merge with the fixed context's attention (normalised O_fix, base-2 LSE L_fix):
    // O = (O_fix 2^(L_fix - M) + o 2^(m sl2 - M)) / (2^(L_fix - M) + l 2^(m sl2 - M))
    float inv = (qv && l > 0.f) ? 1.f / l : 0.f, wfix = 0.f;
    const float* fo = nullptr;
    if (a.fix_o && qv) {
      const long long ft = static_cast<long long>(h) * img_hs + tok;
      const float lf = a.fix_lse[ft];
      const float md = l > 0.f ? m * sl2 : -INFINITY;
      const float mm = fmaxf(lf, md);
      const float wf = ex2(lf - mm), wd = l > 0.f ? ex2(md - mm) : 0.f;
      const float den = wf + l * wd;
      inv = den > 0.f ? wd / den : 0.f;
      wfix = den > 0.f ? wf / den : 0.f;
      fo = a.fix_o + ft * D;
    }
    const float* oc = a.o_comp + (static_cast<long long>(h) * a.R + wr) * D;
    __nv_bfloat16* oi = a.o_img + static_cast<long long>(h) * img_hs * D + tok * D;
    __nv_bfloat16* os = a.o_sel ? a.o_sel + static_cast<long long>(h) * img_hs * D + tok * D : nullptr;
    const float gfix = a.gate_mode == 1 ? 1.f : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t ov[32], gv[32];
      if (ok) {
        tmem_ld32(tO + c0, ov);
        if (learned && gok) tmem_ld32(tS + c0, gv);
        tmem_wait_ld();
      }
      uint32_t po[16], ps[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float s0 = ok ? __uint_as_float(ov[e]) * inv : 0.f, s1 = ok ? __uint_as_float(ov[e + 1]) * inv : 0.f;
        if (fo) {
          const float2 of = __ldg(reinterpret_cast<const float2*>(fo + c0 + e));
          s0 = fmaf(of.x, wfix, s0);
          s1 = fmaf(of.y, wfix, s1);
        }
        float g0 = gfix, g1 = gfix;
        if (learned) {
          g0 = gok ? sigmoid_tanh(__uint_as_float(gv[e])) : 0.f;
          g1 = gok ? sigmoid_tanh(__uint_as_float(gv[e + 1])) : 0.f;
        }
        // g = 0 (selection only, or no compressed value) never reads O'_comp
        const float2 cv = (a.gate_mode == 2 || !qv) ? make_float2(0.f, 0.f)
                                                    : __ldg(reinterpret_cast<const float2*>(oc + c0 + e));
        const float out0 = qv ? g0 * cv.x + (1.f - g0) * s0 : 0.f;
        const float out1 = qv ? g1 * cv.y + (1.f - g1) * s1 : 0.f;
        po[e >> 1] = pack_bf16(out0, out1);
        ps[e >> 1] = pack_bf16(qv ? s0 : 0.f, qv ? s1 : 0.f);
      }
      if (in_grp) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          *reinterpret_cast<uint4*>(oi + c0 + 2 * e) = make_uint4(po[e], po[e + 1], po[e + 2], po[e + 3]);
          if (os) *reinterpret_cast<uint4*>(os + c0 + 2 * e) = make_uint4(ps[e], ps[e + 1], ps[e + 2], ps[e + 3]);
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

cudaError_t launch_sel_union(const SelTcArgs& a, cudaStream_t st) {
  if (a.emax > SEL_UNION_MAX || a.topk * SEL_GROUP > a.emax) return cudaErrorInvalidValue;
  dim3 grid(a.NG, a.H);
  sel_union_kernel<<<grid, 256, 0, st>>>(a);
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
  const int sm = smem_bytes(a.emax);
  cudaError_t e = cudaFuncSetAttribute(sel_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  dim3 grid(a.NG, a.H);
  sel_tc_kernel<<<grid, NTHREADS, sm, st>>>(maps[0], maps[1], maps[2], maps[3], a);
  return cudaGetLastError();
}

}  // namespace gsa
