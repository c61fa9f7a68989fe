// K3: selection-branch attention.
//
// "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (Paper-Notes,
// CVPR 2026), selection branch: for each compressed query the top-k regions
// are chosen from S_guide, their full-resolution K/V tokens are gathered, and
// O_sel = Attention(Q_img, K_sel, V_sel); the queries of one compression
// window share one KV set.  For the VGGT adaptation ("Speed3R-VGGT 适配") the
// key set also holds a fixed global context: every token of the reference
// frame and of the frames sampled every 100 frames.
//
// bf16 path (with the K4 epilogue fused in: O_img is written directly): one
// warp per window (s*s <= 16 queries fill one m16 MMA tile; s = 8 takes four
// warps per window, one per 16 queries);
// 4 windows per CTA, neighbours in raster order so their overlapping region
// choices meet in L2.  Each warp gathers its keys 32 at a time (the tokens of
// the selected regions, then the fixed context) into its own double-buffered
// shared-memory stage with 16-byte cp.async, and runs S = Q K^T, an online
// softmax and O += P V on m16n8k16 MMAs.  Pad keys are masked, pad queries
// write 0.
//
// fp32 path: one thread per query token with fp32 FMA (tiny configs).
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

constexpr int SEL_BN = 32;                     // keys per stage
constexpr int SEL_TILE = SEL_BN * 128;         // bytes of one K (or V) stage
constexpr int SEL_WARP_SMEM = (16 * 128 + 2 * 2 * SEL_TILE + KC_MAX * 8 + 2 * SEL_BN + 127) / 128 * 128;
constexpr int SEL_WARPS = 4;

// Geometry of one selected region: .x = flat token index (within the head) of
// its top-left token, .y = (valid rows << 16) | valid cols, both capped at S.
template <int S>
__device__ __forceinline__ int2 region_base(const SelArgs& a, int reg) {
  const int f = reg / a.rpf, rr = reg - f * a.rpf;
  const int rx = a.g.Wp / S;
  const int i = rr / rx, j = rr - i * rx;
  const int ly = min(a.g.Hv - i * S, S), lx = min(a.g.Wv - j * S, S);
  return make_int2((f * a.g.Hp + i * S) * a.g.Wp + j * S, (ly << 16) | lx);
}

// Source of key position p of a window's key list: the s*s tokens of each
// selected region in order (regions described by `rb`), then per fixed frame
// its special tokens and its padded image grid.  Returns false for pad tokens
// and positions past the end.
template <int S>
__device__ __forceinline__ bool key_src(const SelArgs& a, const int2* rb, int p, int nk_dyn,
                                        int nkeys, long long& off, bool& spec) {
  spec = false;
  off = 0;
  if (p < nk_dyn) {
    const int slot = p / (S * S), tq = p % (S * S);
    const int2 r = rb[slot];
    const int dy = tq / S, dx = tq % S;
    off = r.x + dy * a.g.Wp + dx;
    return dy < (r.y >> 16) && dx < (r.y & 0xffff);
  }
  if (p >= nkeys) return false;
  const int per = a.g.ns + a.g.Hp * a.g.Wp;
  const int pf = p - nk_dyn;
  const int fi = pf / per, o = pf - fi * per;
  int frame = 0;
  for (int i = 0; i < a.n_fixed; ++i)
    if (i == fi) frame = a.fixed[i];
  if (o < a.g.ns) {
    spec = true;
    off = static_cast<long long>(frame) * a.g.ns + o;
    return true;
  }
  off = static_cast<long long>(frame) * a.g.Hp * a.g.Wp + (o - a.g.ns);
  return a.g.img_valid(o - a.g.ns);
}

__device__ __forceinline__ float sigmoid_fast(float x) {
  const float e = ex2(fminf(-x * LOG2E, 126.f));
  return __fdividef(1.f, 1.f + e);
}

// GATE: the window's outputs go straight through the K4 epilogue (nearest
// upsample of O'_comp, g = sigmoid(W_g q), blend) and O_img is written; O_sel
// itself is written only when a.o_sel is set.  G = Q W_g^T reuses the
// window's Q fragments; W_g's B fragments are 32-bit loads of its rows (L1);
// g is computed before the key loop and held as bf16 pairs (relative error
// 2^-9 of g, below the bf16 rounding of the output).
template <int S, bool GATE>
__global__ void __launch_bounds__(SEL_WARPS * 32) sel_kernel_bf16(const SelArgs a, const EpiArgs ep) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, lr = lane & 7;
  uint8_t* wbase = smem + warp * SEL_WARP_SMEM;
  const uint32_t sQ = smem_u32(wbase);
  const uint32_t sKV = sQ + 16 * 128;
  int2* sReg = reinterpret_cast<int2*>(wbase + 16 * 128 + 4 * SEL_TILE);
  uint8_t* sValid = reinterpret_cast<uint8_t*>(sReg + KC_MAX);

  // RB row blocks of 16 queries per window.  s = 8: the CTA's four warps take
  // one window, 16 queries each; they gather its keys together into the first
  // warp's stages (8 keys per warp and block) and synchronise per block.
  constexpr int RB = (S * S + 15) / 16;
  constexpr bool SH = RB > 1;
  static_assert(!SH || RB == SEL_WARPS, "one window per CTA");
  const uint32_t sKVs = SH ? smem_u32(smem) + 16 * 128 : sKV;
  uint8_t* sValidS = SH ? reinterpret_cast<uint8_t*>(reinterpret_cast<int2*>(smem + 16 * 128 + 4 * SEL_TILE) + KC_MAX)
                        : sValid;
  auto stage_sync = [&]() {
    if constexpr (SH) __syncthreads(); else __syncwarp();
  };
  const long long wq = static_cast<long long>(blockIdx.x) * SEL_WARPS + warp;
  const long long win = wq / RB;
  const int rb = static_cast<int>(wq - win * RB);
  if (win >= static_cast<long long>(a.H) * a.R) return;      // warp-uniform
  const int h = static_cast<int>(win / a.R);
  const int r = static_cast<int>(win - static_cast<long long>(h) * a.R);
  const long long img_hs = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp * D;
  const long long spec_hs = static_cast<long long>(a.F) * a.g.ns * D;
  const __nv_bfloat16* qh = reinterpret_cast<const __nv_bfloat16*>(a.q_img) + h * img_hs;
  const __nv_bfloat16* kh = reinterpret_cast<const __nv_bfloat16*>(a.k_img) + h * img_hs;
  const __nv_bfloat16* vh = reinterpret_cast<const __nv_bfloat16*>(a.v_img) + h * img_hs;
  const __nv_bfloat16* ksh = reinterpret_cast<const __nv_bfloat16*>(a.k_spec) + h * spec_hs;
  const __nv_bfloat16* vsh = reinterpret_cast<const __nv_bfloat16*>(a.v_spec) + h * spec_hs;

  // window geometry
  const int f = r / a.rpf, rr0 = r - f * a.rpf;
  const int rx = a.g.Wp / S;
  const int wi = rr0 / rx, wj = rr0 - wi * rx;

  // selected regions of this window
  for (int j = lane; j < a.topk; j += 32) {
    int v = a.idx[win * a.topk + j];
    if (v < 0 || v >= a.R) {
      set_error(a.err, ERR_BOUNDS);
      v = 0;
    }
    sReg[j] = region_base<S>(a, v);
  }
  // queries: token q = (a_, b_) of the window, rows >= s*s are zero
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int e = lane + 32 * it;
    const int row = e >> 3, c = e & 7;
    const int qr = 16 * rb + row;                  // query of the window
    const int y = wi * S + qr / S, x = wj * S + qr % S;
    const bool ok = qr < S * S && y < a.g.Hv && x < a.g.Wv;
    const long long tok = ok ? (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x : 0;
    cp_async16(sQ + swz(row, c), qh + tok * D + c * 8, ok ? 16 : 0);
  }
  cp_async_commit();
  __syncwarp();

  const int nk_dyn = a.topk * S * S;
  // the fixed context, when computed apart (a.fix_o), is merged at the end instead
  const int nkeys = nk_dyn + (a.fix_o ? 0 : a.n_fixed * (a.g.ns + a.g.Hp * a.g.Wp));
  const int nblk = (nkeys + SEL_BN - 1) / SEL_BN;

  // each lane resolves one key of the block (the warp's 32, or 8 with s = 8)
  // and hands its source to the 8 lanes that copy that key's 128-byte row:
  // src >= 0 image token, src <= -2 special token -(src + 2), -1 no key
  auto issue = [&](int blk, int st) {
    const uint32_t sK = sKVs + st * 2 * SEL_TILE;
    const uint32_t sV = sK + SEL_TILE;
    constexpr int NKW = SH ? 8 : 32;              // keys this warp copies per block
    const int kbase = SH ? 8 * warp : 0;
    long long mine = -1;
    if (lane < NKW) {
      long long off;
      bool spec;
      if (key_src<S>(a, sReg, blk * SEL_BN + kbase + lane, nk_dyn, nkeys, off, spec)) mine = spec ? -(off + 2) : off;
      sValidS[st * SEL_BN + kbase + lane] = mine != -1 ? 1 : 0;
    }
#pragma unroll
    for (int it = 0; it < NKW / 4; ++it) {
      const int local = (lane >> 3) + 4 * it, c = lane & 7;
      const long long src = __shfl_sync(0xffffffffu, mine, local);
      const bool ok = src != -1;
      const bool spec = src <= -2;
      const long long off = spec ? -(src + 2) : (ok ? src : 0);
      const int key = kbase + local;
      cp_async16(sK + swz(key, c), (spec ? ksh : kh) + off * D + c * 8, ok ? 16 : 0);
      cp_async16(sV + swz(key, c), (spec ? vsh : vh) + off * D + c * 8, ok ? 16 : 0);
    }
  };

  issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncwarp();                                   // this warp's Q
  uint32_t qf[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(sQ + swz(lr + 8 * (mi & 1), 2 * ks + (mi >> 1)), qf[ks][0], qf[ks][1], qf[ks][2],
            qf[ks][3]);

  // gate (fused epilogue): g = sigmoid(Q W_g^T) now, while the first keys are
  // in flight; kept as bf16 pairs (channel pair of each accumulator element)
  uint32_t gp[8][2];
  if constexpr (GATE) {
    const float gfix = ep.gate_mode == 1 ? 1.f : 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) gp[nt][0] = gp[nt][1] = pack_bf16(gfix, gfix);
    if (ep.gate_mode == 0) {
      const __nv_bfloat16* wg = reinterpret_cast<const __nv_bfloat16*>(ep.w_g) + static_cast<long long>(h) * D * D;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float ga[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const __nv_bfloat16* wr = wg + (8 * nt + g) * D + 16 * ks + 2 * t;
          const uint32_t b0 = __ldg(reinterpret_cast<const unsigned int*>(wr));
          const uint32_t b1 = __ldg(reinterpret_cast<const unsigned int*>(wr + 8));
          mma_bf16(ga, qf[ks], b0, b1);
        }
        gp[nt][0] = pack_bf16(sigmoid_fast(ga[0]), sigmoid_fast(ga[1]));
        gp[nt][1] = pack_bf16(sigmoid_fast(ga[2]), sigmoid_fast(ga[3]));
      }
    }
  }

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};
  const float sl2 = a.scale_log2;

  for (int blk = 0; blk < nblk; ++blk) {
    const int st = blk & 1;
    stage_sync();                                 // every reader is done with stage st^1
    if (blk + 1 < nblk) issue(blk + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    stage_sync();                                 // every writer's part of stage st has landed
    const uint32_t sK = sKVs + st * 2 * SEL_TILE;
    const uint32_t sV = sK + SEL_TILE;

    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (!sValidS[st * SEL_BN + 8 * nt + 2 * t + e]) {
          s[nt][e] = -INFINITY;
          s[nt][2 + e] = -INFINITY;
        }

#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * rr], s[nt][2 * rr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m[rr], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2((m[rr] - m_use) * sl2);
      l[rr] *= alpha;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        o[nt][2 * rr] *= alpha;
        o[nt][2 * rr + 1] *= alpha;
      }
      const float mb = m_use * sl2;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float p0 = ex2(fmaf(s[nt][2 * rr], sl2, -mb));
        const float p1 = ex2(fmaf(s[nt][2 * rr + 1], sl2, -mb));
        s[nt][2 * rr] = p0;
        s[nt][2 * rr + 1] = p1;
        l[rr] += p0 + p1;
      }
      m[rr] = m_new;
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(16 * kk + lr + 8 * (mi & 1), 2 * dp + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa, b0, b1);
        mma_bf16(o[2 * dp + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  __nv_bfloat16* oh = a.o_sel ? reinterpret_cast<__nv_bfloat16*>(a.o_sel) + h * img_hs : nullptr;
  __nv_bfloat16* ih = GATE ? reinterpret_cast<__nv_bfloat16*>(ep.o_img) + h * img_hs : nullptr;
  const float* cr = GATE ? ep.o_comp + (static_cast<long long>(h) * a.R + r) * D : nullptr;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 1);
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 2);
    const int qr = 16 * rb + g + 8 * rr;           // query of the window
    if (qr >= S * S) continue;
    const int y = wi * S + qr / S, x = wj * S + qr % S;
    const bool qv = y < a.g.Hv && x < a.g.Wv;
    const long long tok = (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x;
    // merge with the fixed context's attention (normalised O_fix, base-2 LSE L_fix):
    // O = (O_fix 2^(L_fix - M) + o 2^(m sl2 - M)) / (2^(L_fix - M) + l 2^(m sl2 - M))
    float inv = (qv && l[rr] > 0.f) ? 1.f / l[rr] : 0.f, wfix = 0.f;
    const float* fo = nullptr;
    if (a.fix_o && qv) {
      const long long ft = static_cast<long long>(h) * a.F * a.g.Hp * a.g.Wp + tok;
      const float lf = a.fix_lse[ft];
      const float md = l[rr] > 0.f ? m[rr] * sl2 : -INFINITY;
      const float mm = fmaxf(lf, md);
      const float wf = ex2(lf - mm), wd = l[rr] > 0.f ? ex2(md - mm) : 0.f;
      const float den = wf + l[rr] * wd;
      inv = den > 0.f ? wd / den : 0.f;
      wfix = den > 0.f ? wf / den : 0.f;
      fo = a.fix_o + ft * D;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = 8 * nt + 2 * t;
      float s0 = o[nt][2 * rr] * inv, s1 = o[nt][2 * rr + 1] * inv;
      if (fo) {
        const float2 of = __ldg(reinterpret_cast<const float2*>(fo + c));
        s0 = fmaf(of.x, wfix, s0);
        s1 = fmaf(of.y, wfix, s1);
      }
      if (oh) *reinterpret_cast<uint32_t*>(oh + tok * D + c) = pack_bf16(s0, s1);
      if constexpr (GATE) {
        float out0 = 0.f, out1 = 0.f;
        if (qv) {
          const float2 gg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gp[nt][rr]));
          const float g0 = gg.x, g1 = gg.y;
          // g = 0 (no compressed value) never reads O'_comp, which may not exist
          const float2 oc = ep.gate_mode == 2 ? make_float2(0.f, 0.f) : __ldg(reinterpret_cast<const float2*>(cr + c));
          out0 = g0 * oc.x + (1.f - g0) * s0;
          out1 = g1 * oc.y + (1.f - g1) * s1;
        }
        *reinterpret_cast<uint32_t*>(ih + tok * D + c) = pack_bf16(out0, out1);
      }
    }
  }
}

// fp32: one thread per query token
template <int S>
__global__ void __launch_bounds__(128) sel_kernel_f32(const SelArgs a) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long per_head = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
  if (tid >= per_head * a.H) return;
  const int h = static_cast<int>(tid / per_head);
  const long long n = tid - h * per_head;
  const int f = static_cast<int>(n / (a.g.Hp * a.g.Wp));
  const int o2 = static_cast<int>(n - static_cast<long long>(f) * a.g.Hp * a.g.Wp);
  const int y = o2 / a.g.Wp, x = o2 - y * a.g.Wp;
  const long long img_hs = per_head * D;
  const long long spec_hs = static_cast<long long>(a.F) * a.g.ns * D;
  float* out = reinterpret_cast<float*>(a.o_sel) + h * img_hs + n * D;
  if (y >= a.g.Hv || x >= a.g.Wv) {
    for (int d = 0; d < D; ++d) out[d] = 0.f;
    return;
  }
  const int r = f * a.rpf + (y / S) * (a.g.Wp / S) + x / S;
  const int* idx = a.idx + (static_cast<long long>(h) * a.R + r) * a.topk;
  for (int j = 0; j < a.topk; ++j)
    if (idx[j] < 0 || idx[j] >= a.R) {
      set_error(a.err, ERR_BOUNDS);
      for (int d = 0; d < D; ++d) out[d] = 0.f;
      return;
    }
  const float* q = reinterpret_cast<const float*>(a.q_img) + h * img_hs + n * D;
  const float* kh = reinterpret_cast<const float*>(a.k_img) + h * img_hs;
  const float* vh = reinterpret_cast<const float*>(a.v_img) + h * img_hs;
  const float* ksh = reinterpret_cast<const float*>(a.k_spec) + h * spec_hs;
  const float* vsh = reinterpret_cast<const float*>(a.v_spec) + h * spec_hs;
  float qr[D], acc[D];
  for (int d = 0; d < D; ++d) { qr[d] = q[d]; acc[d] = 0.f; }
  const int nk_dyn = a.topk * S * S;
  const int nkeys = nk_dyn + a.n_fixed * (a.g.ns + a.g.Hp * a.g.Wp);
  const float scale = a.scale_log2 / LOG2E;
  float mx = -INFINITY, l = 0.f;
  for (int p = 0; p < nkeys; ++p) {
    long long off;
    bool spec;
    bool ok;
    if (p < nk_dyn) {
      const int2 rb = region_base<S>(a, idx[p / (S * S)]);
      ok = key_src<S>(a, &rb, p % (S * S), S * S, S * S, off, spec);
    } else {
      ok = key_src<S>(a, nullptr, p, nk_dyn, nkeys, off, spec);
    }
    if (!ok) continue;
    const float* kp = (spec ? ksh : kh) + off * D;
    const float* vp = (spec ? vsh : vh) + off * D;
    float sc = 0.f;
    for (int d = 0; d < D; ++d) sc = fmaf(qr[d], kp[d], sc);
    sc *= scale;
    const float mn = fmaxf(mx, sc);
    const float al = expf(mx - mn);
    const float pw = expf(sc - mn);
    l = l * al + pw;
    for (int d = 0; d < D; ++d) acc[d] = acc[d] * al + pw * vp[d];
    mx = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  for (int d = 0; d < D; ++d) out[d] = acc[d] * inv;
}

template <int S>
cudaError_t launch_sel_s(const SelArgs& a, bool fp32, cudaStream_t st) {
  if (fp32) {
    const long long n = static_cast<long long>(a.H) * a.F * a.g.Hp * a.g.Wp;
    sel_kernel_f32<S><<<static_cast<unsigned>((n + 127) / 128), 128, 0, st>>>(a);
  } else {
    const int sm = SEL_WARPS * SEL_WARP_SMEM;
    cudaError_t e = cudaFuncSetAttribute(sel_kernel_bf16<S, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    const long long w = static_cast<long long>(a.H) * a.R * ((S * S + 15) / 16);
    EpiArgs none;
    memset(&none, 0, sizeof(none));
    sel_kernel_bf16<S, false><<<static_cast<unsigned>((w + SEL_WARPS - 1) / SEL_WARPS), SEL_WARPS * 32, sm, st>>>(a, none);
  }
  return cudaGetLastError();
}

template <int S>
cudaError_t launch_sel_fused_s(const SelArgs& a, const EpiArgs& ep, cudaStream_t st) {
  const int sm = SEL_WARPS * SEL_WARP_SMEM;
  cudaError_t e = cudaFuncSetAttribute(sel_kernel_bf16<S, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  const long long w = static_cast<long long>(a.H) * a.R * ((S * S + 15) / 16);
  sel_kernel_bf16<S, true><<<static_cast<unsigned>((w + SEL_WARPS - 1) / SEL_WARPS), SEL_WARPS * 32, sm, st>>>(a, ep);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sel_fused(const SelArgs& a, const EpiArgs& ep, cudaStream_t st) {
  switch (a.s) {
    case 1: return launch_sel_fused_s<1>(a, ep, st);
    case 2: return launch_sel_fused_s<2>(a, ep, st);
    case 4: return launch_sel_fused_s<4>(a, ep, st);
    case 8: return launch_sel_fused_s<8>(a, ep, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sel(const SelArgs& a, bool fp32, cudaStream_t st) {
  switch (a.s) {
    case 1: return launch_sel_s<1>(a, fp32, st);
    case 2: return launch_sel_s<2>(a, fp32, st);
    case 4: return launch_sel_s<4>(a, fp32, st);
    case 8: return launch_sel_s<8>(a, fp32, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gsa

// ---- backward: selection branch and gate, one warp per window (s <= 4) ----------
// Per-warp shared memory: Q (2 KB) | 2 stages x (K 4 KB | V 4 KB) | dO_sel tile
// (2 KB, bf16, swizzled) | dS^T and P^T tiles ([32 keys][16 queries] bf16) |
// region table | key validity.
namespace gsa {
namespace {

constexpr int SB_Q = 0;
constexpr int SB_KV = 16 * 128;
constexpr int SB_DO = SB_KV + 4 * SEL_TILE;
constexpr int SB_DST = SB_DO + 16 * 128;
constexpr int SB_PT = SB_DST + SEL_BN * 32;
constexpr int SB_REG = SB_PT + SEL_BN * 32;
constexpr int SB_VAL = SB_REG + KC_MAX * 8;
constexpr int SB_WARP = (SB_VAL + 2 * SEL_BN + 63) / 64 * 64;
// windows (warps) per CTA of the backward: two CTAs of five warps fit the 228 KB
// of shared memory per SM (23,104 bytes per warp; with 128-byte rounding they do not)
constexpr int SB_WARPS = 5;

// A fragments (m16 x k16) of rows [r0, r0 + 16) of a [rows][16] bf16 tile with a 32-byte pitch
__device__ __forceinline__ void ldsm_pitch32(uint32_t base, int r0, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31, j = lane >> 3;
  const uint32_t addr = base + (r0 + (j & 1) * 8 + (lane & 7)) * 32 + (j >> 1) * 16;
  ldsm_x4(addr, a[0], a[1], a[2], a[3]);
}

// four consecutive floats added to global memory in one vector reduction (16-byte aligned)
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// FSPLIT: the forward attended the fixed context apart (s.fix_o set); this kernel then
// loops only the selected regions and leaves the fixed keys to the dense backward
template <int S, bool FSPLIT>
__device__ __forceinline__ void sel_bwd_body(const SelBwdArgs& b) {
  const SelArgs& a = b.s;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, lr = lane & 7;
  uint8_t* wbase = smem + warp * SB_WARP;
  const uint32_t sQ = smem_u32(wbase) + SB_Q;
  const uint32_t sKV = smem_u32(wbase) + SB_KV;
  const uint32_t sdO = smem_u32(wbase) + SB_DO;
  __nv_bfloat16* sdSt = reinterpret_cast<__nv_bfloat16*>(wbase + SB_DST);
  __nv_bfloat16* sPt = reinterpret_cast<__nv_bfloat16*>(wbase + SB_PT);
  int2* sReg = reinterpret_cast<int2*>(wbase + SB_REG);
  uint8_t* sValid = wbase + SB_VAL;

  // a window of s*s queries is RB blocks of 16 rows, one warp each (s = 8: four)
  constexpr int RB = (S * S + 15) / 16;
  const long long wrb = static_cast<long long>(blockIdx.x) * SB_WARPS + warp;
  if (wrb >= static_cast<long long>(a.H) * a.R * RB) return;   // warp-uniform
  const long long win = wrb / RB;
  const int q0 = 16 * static_cast<int>(wrb - win * RB);       // the warp's first query of the window
  const int h = static_cast<int>(win / a.R);
  const int r = static_cast<int>(win - static_cast<long long>(h) * a.R);
  const long long img_hs = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp * D;
  const long long spec_hs = static_cast<long long>(a.F) * a.g.ns * D;
  const __nv_bfloat16* qh = reinterpret_cast<const __nv_bfloat16*>(a.q_img) + h * img_hs;
  const __nv_bfloat16* kh = reinterpret_cast<const __nv_bfloat16*>(a.k_img) + h * img_hs;
  const __nv_bfloat16* vh = reinterpret_cast<const __nv_bfloat16*>(a.v_img) + h * img_hs;
  const __nv_bfloat16* ksh = reinterpret_cast<const __nv_bfloat16*>(a.k_spec) + h * spec_hs;
  const __nv_bfloat16* vsh = reinterpret_cast<const __nv_bfloat16*>(a.v_spec) + h * spec_hs;
  const int f = r / a.rpf, rr0 = r - f * a.rpf;
  const int rx = a.g.Wp / S;
  const int wi = rr0 / rx, wj = rr0 - wi * rx;
  for (int j = lane; j < a.topk; j += 32) {
    int v = a.idx[win * a.topk + j];
    if (v < 0 || v >= a.R) {
      set_error(a.err, ERR_BOUNDS);
      v = 0;
    }
    sReg[j] = region_base<S>(a, v);
  }
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int e = lane + 32 * it;
    const int lrow = e >> 3, c = e & 7, row = q0 + lrow;
    const int y = wi * S + row / S, x = wj * S + row % S;
    const bool ok = row < S * S && y < a.g.Hv && x < a.g.Wv;
    const long long tok = ok ? (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x : 0;
    cp_async16(sQ + swz(lrow, c), qh + tok * D + c * 8, ok ? 16 : 0);
  }
  cp_async_commit();
  __syncwarp();
  const int nk_dyn = a.topk * S * S;
  // with the fixed context computed apart only the selected regions are looped here
  constexpr bool fsplit = FSPLIT;
  const int nkeys = nk_dyn + (fsplit ? 0 : a.n_fixed * (a.g.ns + a.g.Hp * a.g.Wp));
  const int nblk = (nkeys + SEL_BN - 1) / SEL_BN;
  auto issue = [&](int blk, int st) {               // one key per lane, rows copied by 8 lanes
    const uint32_t sK = sKV + st * 2 * SEL_TILE;
    const uint32_t sV = sK + SEL_TILE;
    long long mine = -1;
    {
      long long off;
      bool spec;
      if (key_src<S>(a, sReg, blk * SEL_BN + lane, nk_dyn, nkeys, off, spec)) mine = spec ? -(off + 2) : off;
      sValid[st * SEL_BN + lane] = mine != -1 ? 1 : 0;
    }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int key = (lane >> 3) + 4 * it, c = lane & 7;
      const long long src = __shfl_sync(0xffffffffu, mine, key);
      const bool ok = src != -1;
      const bool spec = src <= -2;
      const long long off = spec ? -(src + 2) : (ok ? src : 0);
      cp_async16(sK + swz(key, c), (spec ? ksh : kh) + off * D + c * 8, ok ? 16 : 0);
      cp_async16(sV + swz(key, c), (spec ? vsh : vh) + off * D + c * 8, ok ? 16 : 0);
    }
  };
  const float sl2 = a.scale_log2;
  const float scale = a.scale_log2 / LOG2E;

  // ---- pass 1: the forward again (online softmax), for O_sel and the row log-sum-exp
  issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncwarp();
  uint32_t qf[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(sQ + swz(lr + 8 * (mi & 1), 2 * ks + (mi >> 1)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  for (int blk = 0; blk < nblk; ++blk) {
    const int st = blk & 1;
    __syncwarp();
    if (blk + 1 < nblk) issue(blk + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const uint32_t sK = sKV + st * 2 * SEL_TILE, sV = sK + SEL_TILE;
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (!sValid[st * SEL_BN + 8 * nt + 2 * t + e]) s[nt][e] = s[nt][2 + e] = -INFINITY;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * rr], s[nt][2 * rr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m[rr], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2((m[rr] - m_use) * sl2);
      l[rr] *= alpha;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        o[nt][2 * rr] *= alpha;
        o[nt][2 * rr + 1] *= alpha;
      }
      const float mb = m_use * sl2;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float p0 = ex2(fmaf(s[nt][2 * rr], sl2, -mb));
        const float p1 = ex2(fmaf(s[nt][2 * rr + 1], sl2, -mb));
        s[nt][2 * rr] = p0;
        s[nt][2 * rr + 1] = p1;
        l[rr] += p0 + p1;
      }
      m[rr] = m_new;
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(16 * kk + lr + 8 * (mi & 1), 2 * dp + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa, b0, b1);
        mma_bf16(o[2 * dp + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  __syncwarp();

  // ---- gate backward and the window's upsample backward --------------------------
  bool qv[2];
  long long tok[2];
  float lse[2], inv[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 1);
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 2);
    const int row = q0 + g + 8 * rr;
    const int y = wi * S + row / S, x = wj * S + row % S;
    qv[rr] = row < S * S && y < a.g.Hv && x < a.g.Wv && l[rr] > 0.f;
    tok[rr] = (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x;
    inv[rr] = qv[rr] ? 1.f / l[rr] : 0.f;
    lse[rr] = qv[rr] ? m[rr] * sl2 + __log2f(l[rr]) : INFINITY;   // +inf: P = 0 on pad rows
  }
  if constexpr (fsplit) {
    // the union with the fixed context: lse over both key sets, and O_sel as the
    // weighted sum of the selected regions' and the fixed context's normalised outputs
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float wd = 0.f, wf = 0.f;
      const float* fo = a.fix_o + (static_cast<long long>(h) * a.F * a.g.Hp * a.g.Wp + tok[rr]) * D;
      if (qv[rr]) {
        const float lf = a.fix_lse[static_cast<long long>(h) * a.F * a.g.Hp * a.g.Wp + tok[rr]];
        const float mm = fmaxf(lf, lse[rr]);
        const float lu = mm + __log2f(ex2(lf - mm) + ex2(lse[rr] - mm));
        wd = ex2(lse[rr] - lu);
        wf = ex2(lf - lu);
        lse[rr] = lu;
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float2 of = qv[rr] ? __ldg(reinterpret_cast<const float2*>(fo + 8 * nt + 2 * t)) : make_float2(0.f, 0.f);
        o[nt][2 * rr] = o[nt][2 * rr] * inv[rr] * wd + of.x * wf;
        o[nt][2 * rr + 1] = o[nt][2 * rr + 1] * inv[rr] * wd + of.y * wf;
      }
      inv[rr] = qv[rr] ? 1.f : 0.f;                  // o now holds the normalised O_sel
    }
  }
  float gg[8][4];                                   // g = sigmoid(W_g q) (or the forced gate)
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) gg[nt][0] = gg[nt][1] = gg[nt][2] = gg[nt][3] = 0.f;
  const __nv_bfloat16* wg = reinterpret_cast<const __nv_bfloat16*>(b.w_g) + static_cast<long long>(h) * D * D;
  if (b.gate_mode == 0) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const __nv_bfloat16* wr = wg + (8 * nt + g) * D + 16 * ks + 2 * t;
        mma_bf16(gg[nt], qf[ks], __ldg(reinterpret_cast<const unsigned int*>(wr)),
                 __ldg(reinterpret_cast<const unsigned int*>(wr + 8)));
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) gg[nt][e] = 1.f / (1.f + __expf(-gg[nt][e]));
    }
  } else {
    const float gfix = b.gate_mode == 1 ? 1.f : 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) gg[nt][0] = gg[nt][1] = gg[nt][2] = gg[nt][3] = gfix;
  }
  const __nv_bfloat16* dOh = b.d_o + h * img_hs;
  const float* ocr = b.o_comp + (static_cast<long long>(h) * a.R + r) * D;
  float* dah = b.da + h * img_hs;
  float Dr[2] = {0.f, 0.f};
  float docs[8][2];                                  // column sums of g * dO over the window
  float dq[8][4];                                    // dq_gate / scale, then + dS K
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const float2 oc = __ldg(reinterpret_cast<const float2*>(ocr + 8 * nt + 2 * t));
    docs[nt][0] = docs[nt][1] = 0.f;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float2 dov = make_float2(0.f, 0.f);
      if (qv[rr])
        dov = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dOh + tok[rr] * D + 8 * nt + 2 * t));
      const float d0 = dov.x, d1 = dov.y;
      const float os0 = o[nt][2 * rr] * inv[rr], os1 = o[nt][2 * rr + 1] * inv[rr];
      const float g0 = gg[nt][2 * rr], g1 = gg[nt][2 * rr + 1];
      const float da0 = b.gate_mode == 0 ? d0 * (oc.x - os0) * g0 * (1.f - g0) : 0.f;
      const float da1 = b.gate_mode == 0 ? d1 * (oc.y - os1) * g1 * (1.f - g1) : 0.f;
      docs[nt][0] += g0 * d0;
      docs[nt][1] += g1 * d1;
      const float dos0 = (1.f - g0) * d0, dos1 = (1.f - g1) * d1;
      Dr[rr] += dos0 * os0 + dos1 * os1;
      o[nt][2 * rr] = dos0;                          // o now holds dO_sel
      o[nt][2 * rr + 1] = dos1;
      gg[nt][2 * rr] = da0;                          // gg now holds da
      gg[nt][2 * rr + 1] = da1;
      const int row = q0 + g + 8 * rr;
      if (row < S * S)
        *reinterpret_cast<float2*>(dah + tok[rr] * D + 8 * nt + 2 * t) = make_float2(da0, da1);
    }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    Dr[rr] += __shfl_xor_sync(0xffffffffu, Dr[rr], 1);
    Dr[rr] += __shfl_xor_sync(0xffffffffu, Dr[rr], 2);
  }
  if constexpr (fsplit) {
    // what the dense backward over the fixed keys reads, for every token of the window
    const long long hq = static_cast<long long>(h) * a.F * a.g.Hp * a.g.Wp;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = q0 + g + 8 * rr;
      if (row >= S * S) continue;
      const int y = wi * S + row / S, x = wj * S + row % S;
      const long long tk = (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        *reinterpret_cast<uint32_t*>(b.dosel + (hq + tk) * D + 8 * nt + 2 * t) =
            qv[rr] ? pack_bf16(o[nt][2 * rr], o[nt][2 * rr + 1]) : 0u;
      if (t == 0) {
        b.lse_u[hq + tk] = qv[rr] ? lse[rr] : INFINITY;
        b.Dq[hq + tk] = qv[rr] ? Dr[rr] : 0.f;
      }
    }
  }
  // dO'_comp[r] = sum over the window's valid tokens of g dO (the window is region r);
  // a window of several row blocks adds its blocks' sums into a zeroed buffer
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = docs[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      docs[nt][e] = v;
    }
  if (g == 0) {
    float* dst = b.d_ocomp + (static_cast<long long>(h) * a.R + r) * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if constexpr (RB == 1) {
        *reinterpret_cast<float2*>(dst + 8 * nt + 2 * t) = make_float2(docs[nt][0], docs[nt][1]);
      } else {
        atomicAdd(dst + 8 * nt + 2 * t, docs[nt][0]);
        atomicAdd(dst + 8 * nt + 2 * t + 1, docs[nt][1]);
      }
    }
  }
  // dq from the gate: dq[k] = sum_c da[c] W_g[c][k] (B fragments from W_g's columns)
#pragma unroll
  for (int i = 0; i < 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  if (b.gate_mode == 0) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t aa[4];
      aa[0] = pack_bf16(gg[2 * kk][0], gg[2 * kk][1]);
      aa[1] = pack_bf16(gg[2 * kk][2], gg[2 * kk][3]);
      aa[2] = pack_bf16(gg[2 * kk + 1][0], gg[2 * kk + 1][1]);
      aa[3] = pack_bf16(gg[2 * kk + 1][2], gg[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int n = 8 * nt + g, k0 = 16 * kk + 2 * t;
        const unsigned short* w16 = reinterpret_cast<const unsigned short*>(wg);
        const uint32_t b0 = static_cast<uint32_t>(__ldg(w16 + k0 * D + n)) |
                            (static_cast<uint32_t>(__ldg(w16 + (k0 + 1) * D + n)) << 16);
        const uint32_t b1 = static_cast<uint32_t>(__ldg(w16 + (k0 + 8) * D + n)) |
                            (static_cast<uint32_t>(__ldg(w16 + (k0 + 9) * D + n)) << 16);
        mma_bf16(dq[nt], aa, b0, b1);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[i][e] /= scale;
  }
  // dO_sel: A fragments and a swizzled bf16 tile (B operand of dV = P^T dO_sel)
  uint32_t dof[4][4];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    dof[kk][0] = pack_bf16(o[2 * kk][0], o[2 * kk][1]);
    dof[kk][1] = pack_bf16(o[2 * kk][2], o[2 * kk][3]);
    dof[kk][2] = pack_bf16(o[2 * kk + 1][0], o[2 * kk + 1][1]);
    dof[kk][3] = pack_bf16(o[2 * kk + 1][2], o[2 * kk + 1][3]);
  }
  uint8_t* sdOp = wbase + SB_DO;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      *reinterpret_cast<uint32_t*>(sdOp + swz(g + 8 * rr, nt) + 4 * t) = pack_bf16(o[nt][2 * rr], o[nt][2 * rr + 1]);
  __syncwarp();

  // ---- pass 2: dS = P (dP - D); dq += dS K; dK += dS^T q, dV += P^T dO_sel (atomics)
  float* dkh = b.dk + h * img_hs;
  float* dvh = b.dv + h * img_hs;
  float* dksh = b.dk_spec ? b.dk_spec + h * spec_hs : nullptr;
  float* dvsh = b.dv_spec ? b.dv_spec + h * spec_hs : nullptr;
  const uint32_t sdSt_a = smem_u32(sdSt), sPt_a = smem_u32(sPt);
  issue(0, 0);
  cp_async_commit();
  for (int blk = 0; blk < nblk; ++blk) {
    const int st = blk & 1;
    __syncwarp();
    if (blk + 1 < nblk) issue(blk + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const uint32_t sK = sKV + st * 2 * SEL_TILE, sV = sK + SEL_TILE;
    float s[4][4], dp[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
        ldsm_x4(sV + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(dp[2 * np], dof[ks], b0, b1);
        mma_bf16(dp[2 * np + 1], dof[ks], b2, b3);
      }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 8 * nt + 2 * t + (e & 1), rr = e >> 1;
        const float p = sValid[st * SEL_BN + key] ? ex2(fmaf(s[nt][e], sl2, -lse[rr])) : 0.f;
        const float ds = p * (dp[nt][e] - Dr[rr]);
        s[nt][e] = ds;
        const int q = g + 8 * rr;
        sdSt[key * 16 + q] = __float2bfloat16_rn(ds);      // [key][query]
        sPt[key * 16 + q] = __float2bfloat16_rn(p);
      }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp2 = 0; dp2 < 4; ++dp2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sK + swz(16 * kk + lr + 8 * (mi & 1), 2 * dp2 + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(dq[2 * dp2], pa, b0, b1);
        mma_bf16(dq[2 * dp2 + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    // dK and dV of the block's 32 keys, 16 at a time, straight to global memory
#pragma unroll 1
    for (int half = 0; half < 4; ++half) {
      const int mt = half & 1;
      const bool isv = half >= 2;
      uint32_t af[4];
      ldsm_pitch32(isv ? sPt_a : sdSt_a, 16 * mt, af);
      float acc[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
      for (int dp2 = 0; dp2 < 4; ++dp2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t((isv ? sdO : sQ) + swz(lr + 8 * (mi & 1), 2 * dp2 + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(acc[2 * dp2], af, b0, b1);
        mma_bf16(acc[2 * dp2 + 1], af, b2, b3);
      }
      const float mul = isv ? 1.f : scale;
      // lanes t and t^1 hold two columns each of the same four: one shuffle gives the
      // even lane four columns of row g and the odd lane four of row g + 8, so each
      // lane adds one 16-byte vector per n-tile (half the reductions of float2 atomics)
      const int rr = t & 1;
      const int key = 16 * mt + g + 8 * rr;
      float* base = nullptr;
      if (sValid[st * SEL_BN + key]) {
        long long off;
        bool spec;
        key_src<S>(a, sReg, blk * SEL_BN + key, nk_dyn, nkeys, off, spec);
        base = spec ? (isv ? dvsh : dksh) : (isv ? dvh : dkh);
        if (base) base += off * D + 4 * (t >> 1);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float x0 = acc[nt][0] * mul, x1 = acc[nt][1] * mul, y0 = acc[nt][2] * mul, y1 = acc[nt][3] * mul;
        const float o0 = __shfl_xor_sync(0xffffffffu, rr ? x0 : y0, 1);
        const float o1 = __shfl_xor_sync(0xffffffffu, rr ? x1 : y1, 1);
        if (base) red_add_v4(base + 8 * nt, rr ? o0 : x0, rr ? o1 : x1, rr ? y0 : o0, rr ? y1 : o1);
      }
    }
  }
  cp_async_wait<0>();
  // dq of the window's tokens: scale (dS K + dq_gate / scale); pad rows 0
  float* dqh = b.dq + h * img_hs;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = q0 + g + 8 * rr;
    if (row >= S * S) continue;
    const int y = wi * S + row / S, x = wj * S + row % S;
    const bool valid = y < a.g.Hv && x < a.g.Wv;
    const long long tk = (static_cast<long long>(f) * a.g.Hp + y) * a.g.Wp + x;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<float2*>(dqh + tk * D + 8 * nt + 2 * t) =
          valid ? make_float2(dq[nt][2 * rr] * scale, dq[nt][2 * rr + 1] * scale) : make_float2(0.f, 0.f);
  }
}

template <int S>
__global__ void __launch_bounds__(SB_WARPS * 32) sel_bwd_kernel(const SelBwdArgs b) {
  sel_bwd_body<S, false>(b);
}
// the fixed-context split keeps more values live; two CTAs per SM still
template <int S>
__global__ void __launch_bounds__(SB_WARPS * 32, 2) sel_bwd_fix_kernel(const SelBwdArgs b) {
  sel_bwd_body<S, true>(b);
}

template <int S, bool FSPLIT>
cudaError_t launch_sel_bwd_sf(const SelBwdArgs& b, cudaStream_t st) {
  const int sm = SB_WARPS * SB_WARP;
  auto kern = FSPLIT ? sel_bwd_fix_kernel<S> : sel_bwd_kernel<S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  if (e != cudaSuccess) return e;
  const long long w = static_cast<long long>(b.s.H) * b.s.R * ((S * S + 15) / 16);   // warps
  kern<<<static_cast<unsigned>((w + SB_WARPS - 1) / SB_WARPS), SB_WARPS * 32, sm, st>>>(b);
  return cudaGetLastError();
}

template <int S>
cudaError_t launch_sel_bwd_s(const SelBwdArgs& b, cudaStream_t st) {
  if (b.s.fix_o) {
    if (!b.dosel || !b.lse_u || !b.Dq || !b.s.fix_lse) return cudaErrorInvalidValue;
    return launch_sel_bwd_sf<S, true>(b, st);
  }
  return launch_sel_bwd_sf<S, false>(b, st);
}

}  // namespace

cudaError_t launch_sel_bwd(const SelBwdArgs& b, cudaStream_t st) {
  switch (b.s.s) {
    case 1: return launch_sel_bwd_s<1>(b, st);
    case 2: return launch_sel_bwd_s<2>(b, st);
    case 4: return launch_sel_bwd_s<4>(b, st);
    case 8: return launch_sel_bwd_s<8>(b, st);
    default: return cudaErrorInvalidValue;
  }
}

namespace {
// one thread per 16-byte piece of a fixed-context key or value row
__global__ void __launch_bounds__(256) fixed_gather_kernel(const SelArgs a, __nv_bfloat16* kfix,
                                                           __nv_bfloat16* vfix, int per_frame) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(a.H) * a.n_fixed * per_frame;
  if (gid >= rows * 8) return;
  const int c = static_cast<int>(gid & 7);
  const long long row = gid >> 3;                        // h * n_fixed * per_frame + i * per_frame + t
  const int t = static_cast<int>(row % per_frame);
  const long long hi = row / per_frame;
  const int i = static_cast<int>(hi % a.n_fixed);
  const int h = static_cast<int>(hi / a.n_fixed);
  const int f = a.fixed[i];
  const __nv_bfloat16 *ks, *vs;
  if (t < a.g.ns) {
    const long long o = ((static_cast<long long>(h) * a.F + f) * a.g.ns + t) * D;
    ks = reinterpret_cast<const __nv_bfloat16*>(a.k_spec) + o;
    vs = reinterpret_cast<const __nv_bfloat16*>(a.v_spec) + o;
  } else {
    const int u = t - a.g.ns, y = u / a.g.Wv, x = u - y * a.g.Wv;
    const long long o = (((static_cast<long long>(h) * a.F + f) * a.g.Hp + y) * a.g.Wp + x) * D;
    ks = reinterpret_cast<const __nv_bfloat16*>(a.k_img) + o;
    vs = reinterpret_cast<const __nv_bfloat16*>(a.v_img) + o;
  }
  reinterpret_cast<uint4*>(kfix + row * D)[c] = reinterpret_cast<const uint4*>(ks)[c];
  reinterpret_cast<uint4*>(vfix + row * D)[c] = reinterpret_cast<const uint4*>(vs)[c];
}
}  // namespace

namespace {
// one thread per four channels of a fixed-context key row: its dK and dV added to the token
__global__ void __launch_bounds__(256) fixed_scatter_kernel(const SelArgs a, const float* dkfix, const float* dvfix,
                                                            float* dk_img, float* dv_img, float* dk_spec,
                                                            float* dv_spec, int per_frame) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(a.H) * a.n_fixed * per_frame;
  if (gid >= rows * 16) return;
  const int c = static_cast<int>(gid & 15);
  const long long row = gid >> 4;
  const int t = static_cast<int>(row % per_frame);
  const long long hi = row / per_frame;
  const int i = static_cast<int>(hi % a.n_fixed);
  const int h = static_cast<int>(hi / a.n_fixed);
  const int f = a.fixed[i];
  float *kd, *vd;
  if (t < a.g.ns) {
    const long long o = ((static_cast<long long>(h) * a.F + f) * a.g.ns + t) * D;
    kd = dk_spec + o;
    vd = dv_spec + o;
  } else {
    const int u = t - a.g.ns, y = u / a.g.Wv, x = u - y * a.g.Wv;
    const long long o = (((static_cast<long long>(h) * a.F + f) * a.g.Hp + y) * a.g.Wp + x) * D;
    kd = dk_img + o;
    vd = dv_img + o;
  }
  const float4 dk = reinterpret_cast<const float4*>(dkfix + row * D)[c];
  const float4 dv = reinterpret_cast<const float4*>(dvfix + row * D)[c];
  float4 k0 = reinterpret_cast<float4*>(kd)[c], v0 = reinterpret_cast<float4*>(vd)[c];
  k0.x += dk.x; k0.y += dk.y; k0.z += dk.z; k0.w += dk.w;
  v0.x += dv.x; v0.y += dv.y; v0.z += dv.z; v0.w += dv.w;
  reinterpret_cast<float4*>(kd)[c] = k0;
  reinterpret_cast<float4*>(vd)[c] = v0;
}
}  // namespace

cudaError_t launch_fixed_scatter_add(const SelArgs& a, const float* dkfix, const float* dvfix, float* dk_img,
                                     float* dv_img, float* dk_spec, float* dv_spec, cudaStream_t st) {
  const int per_frame = a.g.ns + a.g.Hv * a.g.Wv;
  const long long n = static_cast<long long>(a.H) * a.n_fixed * per_frame * 16;
  if (n <= 0) return cudaSuccess;
  fixed_scatter_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a, dkfix, dvfix, dk_img, dv_img, dk_spec,
                                                                               dv_spec, per_frame);
  return cudaGetLastError();
}

cudaError_t launch_fixed_gather(const SelArgs& a, __nv_bfloat16* kfix, __nv_bfloat16* vfix, cudaStream_t st) {
  const int per_frame = a.g.ns + a.g.Hv * a.g.Wv;
  const long long n = static_cast<long long>(a.H) * a.n_fixed * per_frame * 8;
  if (n <= 0) return cudaSuccess;
  fixed_gather_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a, kfix, vfix, per_frame);
  return cudaGetLastError();
}

}  // namespace gsa
