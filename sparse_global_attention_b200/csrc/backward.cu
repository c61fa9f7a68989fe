// Backward pass of the GSA layer.
//
// The notes train the layer end to end ("Speed3R: Sparse Feed-forward 3D
// Reconstruction Models", Paper-Notes CVPR 2026, GSA core design); the
// backward is the gradient of the forward with the region selection held
// fixed (TopKSelect passes no gradient).  With dO the output gradient:
//   gate       g = sigmoid(W_g q):  dO_sel = (1-g) dO,  dO_comp = g dO,
//              da = dO (O_comp - O_sel) g (1-g),  dq += W_g^T da,  dW_g += da q^T
//   upsample   dO'_comp[r] = sum of dO_comp over the valid tokens of region r
//   attention  (each of compressed, selection, special) with P = softmax(S):
//              D = rowsum(dO o O),  dS = P o (dO V^T - D),
//              dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO
//   pool       each valid token of region r gets dX_comp[r] / |valid tokens of r|
// Kernels:
//   attn_bwd_dq / attn_bwd_dkv  dense attention backward (compressed branch,
//       special tokens), flash style: P is recomputed tile by tile from the
//       forward's log-sum-exp; dQ by query tiles, dK/dV by key tiles, so no
//       gradient needs atomics.  m16n8k16 bf16 MMAs, fp32 accumulation.
//   sel_bwd     one warp per window: recomputes the selection forward, runs the
//       gate backward, writes dO'_comp of its region and dq of its tokens, and
//       adds dK/dV of its keys (shared by many windows) with fp32 atomics.
//   pool_bwd, dwg_kernel, rowdot  the elementwise and reduction steps.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

constexpr int BT = 64;                  // rows per CTA tile (4 warps x 16) and keys/queries per stage
constexpr int TB = BT * 128;            // bytes of a 64 x 64 bf16 tile

// A-operand fragments (m16 x k16, 4 k-steps over d = 64) of the 16 rows of a
// swizzled tile starting at `base`
__device__ __forceinline__ void load_afrag(uint32_t base, uint32_t (&f)[4][4]) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, lr = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(base + swz(lr + 8 * (mi & 1), 2 * ks + (mi >> 1)), f[ks][0], f[ks][1], f[ks][2], f[ks][3]);
}

// acc[16 x 64] += A[16 x 64 (k = d)] . X^T where X is a 64-row tile [n][d]
__device__ __forceinline__ void mma_xt(float (&acc)[8][4], const uint32_t (&a)[4][4], uint32_t xt) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, lr = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(xt + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
      mma_bf16(acc[2 * np], a[ks], b0, b1);
      mma_bf16(acc[2 * np + 1], a[ks], b2, b3);
    }
}

// acc[16 x 64 (d)] += A[16 x 64 (k = rows of X)] . X where X is a 64-row tile [k][d]
__device__ __forceinline__ void mma_x(float (&acc)[8][4], const uint32_t (&a)[4][4], uint32_t x) {
  const int lane = threadIdx.x & 31, mi = lane >> 3, lr = lane & 7;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int dp = 0; dp < 4; ++dp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(x + swz(16 * kk + lr + 8 * (mi & 1), 2 * dp + (mi >> 1)), b0, b1, b2, b3);
      mma_bf16(acc[2 * dp], a[kk], b0, b1);
      mma_bf16(acc[2 * dp + 1], a[kk], b2, b3);
    }
}

// C fragments of a 16 x 64 product as bf16 A fragments (k = its 64 columns)
__device__ __forceinline__ void c_to_a(const float (&c)[8][4], uint32_t (&a)[4][4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    a[kk][0] = pack_bf16(c[2 * kk][0], c[2 * kk][1]);
    a[kk][1] = pack_bf16(c[2 * kk][2], c[2 * kk][3]);
    a[kk][2] = pack_bf16(c[2 * kk + 1][0], c[2 * kk + 1][1]);
    a[kk][3] = pack_bf16(c[2 * kk + 1][2], c[2 * kk + 1][3]);
  }
}

__device__ __forceinline__ void zero(float (&c)[8][4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i][0] = c[i][1] = c[i][2] = c[i][3] = 0.f;
}

// rows [row0, row0 + 64) of a [n][64] bf16 tensor into a swizzled tile; rows past n read zeros
__device__ __forceinline__ void tile_load(uint32_t dst, const __nv_bfloat16* src, long long row0, long long n) {
#pragma unroll
  for (int it = 0; it < (BT * 8) / 128; ++it) {
    const int e = threadIdx.x + it * 128;
    const int r = e >> 3, c = e & 7;
    const bool ok = row0 + r < n;
    cp_async16(dst + swz(r, c), src + (ok ? row0 + r : 0) * D + c * 8, ok ? 16 : 0);
  }
}

// segment and first key of global key tile tt
__device__ __forceinline__ int bseg(const BwdArgs& a, int tt, long long& kb) {
  const int t0 = static_cast<int>((a.n_k[0] + BT - 1) / BT);
  const int seg = (a.nseg > 1 && tt >= t0) ? 1 : 0;
  kb = static_cast<long long>(seg ? tt - t0 : tt) * BT;
  return seg;
}

// ---- dQ: CTA = 64 query rows, loop over every key tile of both segments -------
// smem: Q hi | Q lo | dO | 2 stages x (K hi | K lo | V) | key validity
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(const BwdArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb, sQl = sb + TB, sdO = sb + 2 * TB, sST = sb + 3 * TB;
  constexpr int STG = 3 * TB;
  uint8_t* sVal = smem + 3 * TB + 2 * STG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const long long q0 = static_cast<long long>(blockIdx.x) * BT;
  const bool split = a.q_lo != nullptr;

  tile_load(sQ, a.q + h * a.q_hs, q0, a.n_q);
  if (split) tile_load(sQl, a.q_lo + h * a.q_hs, q0, a.n_q);
  tile_load(sdO, a.dO + h * a.do_hs, q0, a.n_q);
  cp_async_commit();
  const int t0 = static_cast<int>((a.n_k[0] + BT - 1) / BT);
  const int ntile = t0 + (a.nseg > 1 ? static_cast<int>((a.n_k[1] + BT - 1) / BT) : 0);

  auto issue = [&](int tt, int st) {
    long long kb;
    const int seg = bseg(a, tt, kb);
    const uint32_t s = sST + st * STG;
    tile_load(s, a.k[seg] + h * a.kv_hs[seg], kb, a.n_k[seg]);
    if (split && seg == 0) tile_load(s + TB, a.k_lo + h * a.kv_hs[0], kb, a.n_k[0]);
    tile_load(s + 2 * TB, a.v[seg] + h * a.kv_hs[seg], kb, a.n_k[seg]);
    if (threadIdx.x < BT) {
      const long long key = kb + threadIdx.x;
      sVal[st * BT + threadIdx.x] = (key < a.n_k[seg] && key_valid(a.kmask[seg], a.g, key)) ? 1 : 0;
    }
  };
  issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qf[4][4], qlf[4][4], dof[4][4];
  load_afrag(sQ + warp * 16 * 128, qf);
  if (split) load_afrag(sQl + warp * 16 * 128, qlf);
  load_afrag(sdO + warp * 16 * 128, dof);
  float lse[2], Dr[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const long long row = q0 + warp * 16 + g + 8 * rr;
    const bool ok = row < a.n_q;
    lse[rr] = ok ? a.lse2[h * static_cast<long long>(a.n_q) + row] : 0.f;
    Dr[rr] = ok ? a.Dv[h * static_cast<long long>(a.n_q) + row] : 0.f;
  }
  float dq[8][4];
  zero(dq);
  for (int tt = 0; tt < ntile; ++tt) {
    const int st = tt & 1;
    __syncthreads();
    if (tt + 1 < ntile) issue(tt + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    long long kb;
    const int seg = bseg(a, tt, kb);
    const uint32_t sK = sST + st * STG, sKl = sK + TB, sV = sK + 2 * TB;
    float s[8][4], dp[8][4];
    zero(s);
    mma_xt(s, qf, sK);
    if (split && seg == 0) {
      mma_xt(s, qf, sKl);
      mma_xt(s, qlf, sK);
    }
    zero(dp);
    mma_xt(dp, dof, sV);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * nt + 2 * t + (e & 1), rr = e >> 1;
        const float p = sVal[st * BT + col] ? ex2(s[nt][e] * a.scale_log2 - lse[rr]) : 0.f;
        s[nt][e] = p * (dp[nt][e] - Dr[rr]);                  // dS
      }
    uint32_t dsa[4][4];
    c_to_a(s, dsa);
    mma_x(dq, dsa, sK);
  }
  cp_async_wait<0>();
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const long long row = q0 + warp * 16 + g + 8 * rr;
    if (row >= a.n_q) continue;
    float* out = a.dq + h * a.dq_hs + row * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float2 v = make_float2(dq[nt][2 * rr] * a.scale, dq[nt][2 * rr + 1] * a.scale);
      float2* p = reinterpret_cast<float2*>(out + 8 * nt + 2 * t);
      if (a.dq_accum) {
        const float2 o = *p;
        v.x += o.x;
        v.y += o.y;
      }
      *p = v;
    }
  }
}

// ---- dK, dV of one key segment: CTA = 64 keys, loop over every query tile -----
// smem: K hi | K lo | V | 2 stages x (Q hi | Q lo | dO) | 2 x (lse, D) per stage
__global__ void __launch_bounds__(128) attn_bwd_dkv_kernel(const BwdArgs a, int seg) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb, sKl = sb + TB, sV = sb + 2 * TB, sST = sb + 3 * TB;
  constexpr int STG = 3 * TB;
  float* sLD = reinterpret_cast<float*>(smem + 3 * TB + 2 * STG);      // [2 stages][lse 64 | D 64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int h = blockIdx.y;
  const long long k0 = static_cast<long long>(blockIdx.x) * BT;
  const bool split = a.q_lo != nullptr && seg == 0;
  const long long nk = a.n_k[seg];

  tile_load(sK, a.k[seg] + h * a.kv_hs[seg], k0, nk);
  if (split) tile_load(sKl, a.k_lo + h * a.kv_hs[0], k0, nk);
  tile_load(sV, a.v[seg] + h * a.kv_hs[seg], k0, nk);
  cp_async_commit();
  const int ntile = static_cast<int>((a.n_q + BT - 1) / BT);
  auto issue = [&](int qt, int st) {
    const uint32_t s = sST + st * STG;
    const long long q0 = static_cast<long long>(qt) * BT;
    tile_load(s, a.q + h * a.q_hs, q0, a.n_q);
    if (split) tile_load(s + TB, a.q_lo + h * a.q_hs, q0, a.n_q);
    tile_load(s + 2 * TB, a.dO + h * a.do_hs, q0, a.n_q);
    if (threadIdx.x < BT) {
      const long long row = q0 + threadIdx.x;
      const bool ok = row < a.n_q;
      // rows past the end: lse = +inf makes P = 0
      sLD[st * 2 * BT + threadIdx.x] = ok ? a.lse2[h * static_cast<long long>(a.n_q) + row] : INFINITY;
      sLD[st * 2 * BT + BT + threadIdx.x] = ok ? a.Dv[h * static_cast<long long>(a.n_q) + row] : 0.f;
    }
  };
  issue(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t kf[4][4], klf[4][4], vf[4][4];
  load_afrag(sK + warp * 16 * 128, kf);
  if (split) load_afrag(sKl + warp * 16 * 128, klf);
  load_afrag(sV + warp * 16 * 128, vf);
  bool kv[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const long long key = k0 + warp * 16 + g + 8 * rr;
    kv[rr] = key < nk && key_valid(a.kmask[seg], a.g, key);
  }
  float dk[8][4], dv[8][4];
  zero(dk);
  zero(dv);
  for (int qt = 0; qt < ntile; ++qt) {
    const int st = qt & 1;
    __syncthreads();
    if (qt + 1 < ntile) issue(qt + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sQ = sST + st * STG, sQl = sQ + TB, sdO = sQ + 2 * TB;
    const float* lse = sLD + st * 2 * BT;
    const float* Dq = lse + BT;
    float s[8][4], dp[8][4];
    zero(s);
    mma_xt(s, kf, sQ);                       // S^T = K Q^T
    if (split) {
      mma_xt(s, klf, sQ);
      mma_xt(s, kf, sQl);
    }
    zero(dp);
    mma_xt(dp, vf, sdO);                     // dP^T = V dO^T
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * nt + 2 * t + (e & 1), rr = e >> 1;
        const float p = kv[rr] ? ex2(s[nt][e] * a.scale_log2 - lse[col]) : 0.f;
        s[nt][e] = p;                                      // P^T
        dp[nt][e] = p * (dp[nt][e] - Dq[col]);             // dS^T
      }
    uint32_t pa[4][4], dsa[4][4];
    c_to_a(s, pa);
    c_to_a(dp, dsa);
    mma_x(dv, pa, sdO);                      // dV += P^T dO
    mma_x(dk, dsa, sQ);                      // dK += dS^T Q
  }
  cp_async_wait<0>();
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const long long key = k0 + warp * 16 + g + 8 * rr;
    if (key >= nk) continue;
    float* ok_ = a.dk[seg] + h * a.dkv_hs[seg] + key * D;
    float* ov = a.dv[seg] + h * a.dkv_hs[seg] + key * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float2 vk = make_float2(dk[nt][2 * rr] * a.scale, dk[nt][2 * rr + 1] * a.scale);
      float2 vv = make_float2(dv[nt][2 * rr], dv[nt][2 * rr + 1]);
      float2* pk = reinterpret_cast<float2*>(ok_ + 8 * nt + 2 * t);
      float2* pv = reinterpret_cast<float2*>(ov + 8 * nt + 2 * t);
      if (a.dkv_accum) {
        const float2 ak = *pk, av = *pv;
        vk.x += ak.x; vk.y += ak.y;
        vv.x += av.x; vv.y += av.y;
      }
      *pk = vk;
      *pv = vv;
    }
  }
}

}  // namespace

constexpr int DQ_SMEM = 3 * TB + 2 * 3 * TB + 2 * BT;
constexpr int DKV_SMEM = 3 * TB + 2 * 3 * TB + 2 * 2 * BT * 4;

cudaError_t launch_attn_bwd_dkv(const BwdArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM);
  if (e != cudaSuccess) return e;
  for (int seg = 0; seg < a.nseg; ++seg) {
    if (!a.dk[seg]) continue;
    attn_bwd_dkv_kernel<<<dim3(static_cast<unsigned>((a.n_k[seg] + BT - 1) / BT), a.H), 128, DKV_SMEM, st>>>(a, seg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_attn_bwd(const BwdArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DKV_SMEM);
  if (e != cudaSuccess) return e;
  attn_bwd_dq_kernel<<<dim3(static_cast<unsigned>((a.n_q + BT - 1) / BT), a.H), 128, DQ_SMEM, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int seg = 0; seg < a.nseg; ++seg) {
    if (!a.dk[seg]) continue;
    attn_bwd_dkv_kernel<<<dim3(static_cast<unsigned>((a.n_k[seg] + BT - 1) / BT), a.H), 128, DKV_SMEM, st>>>(a, seg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

namespace {

// dX_img[t] += dX_comp[region(t)] / (valid tokens of the region), valid t only
__global__ void __launch_bounds__(256) pool_bwd_kernel(const PoolBwdArgs a) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long per = static_cast<long long>(a.Hp) * a.Wp;
  const long long total = static_cast<long long>(a.H) * a.F * per * (D / 4);
  if (gid >= total) return;
  const int c4 = static_cast<int>(gid % (D / 4));
  const long long tokg = gid / (D / 4);                 // (h*F + f)*per + o
  const int o = static_cast<int>(tokg % per);
  const long long hf = tokg / per;
  const int y = o / a.Wp, x = o - y * a.Wp;
  if (y >= a.Hv || x >= a.Wv) return;
  const int s = a.s, rx = a.Wp / s, rpf = (a.Hp / s) * rx;
  const int i = y / s, j = x / s;
  const int cnt = min(a.Hv - i * s, s) * min(a.Wv - j * s, s);
  const long long h = hf / a.F, f = hf - h * a.F;
  const long long reg = (h * a.F + f) * rpf + static_cast<long long>(i) * rx + j;
  const float inv = 1.f / static_cast<float>(cnt);
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const float4 d = *reinterpret_cast<const float4*>(a.dcomp[q] + reg * D + 4 * c4);
    float4* dst = reinterpret_cast<float4*>(a.dimg[q] + tokg * D + 4 * c4);
    float4 v = *dst;
    v.x += d.x * inv; v.y += d.y * inv; v.z += d.z * inv; v.w += d.w * inv;
    *dst = v;
  }
}

// one warp per row: D = sum dO o O, optional bf16 copy of a fp32 dO
__global__ void __launch_bounds__(256) rowdot_kernel(const float* do32, const __nv_bfloat16* do16, const float* o32,
                                                     const __nv_bfloat16* o16, long long rows, float* Dout,
                                                     __nv_bfloat16* do16_out) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const long long e = row * D + 2 * lane;
  float2 d, o;
  if (do32) d = *reinterpret_cast<const float2*>(do32 + e);
  else d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(do16 + e));
  if (o32) o = *reinterpret_cast<const float2*>(o32 + e);
  else o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o16 + e));
  float v = d.x * o.x + d.y * o.y;
#pragma unroll
  for (int k = 16; k; k >>= 1) v += __shfl_xor_sync(0xffffffffu, v, k);
  if (lane == 0) Dout[row] = v;
  if (do16_out) *reinterpret_cast<uint32_t*>(do16_out + e) = pack_bf16(d.x, d.y);
}

// dW_g[h][c][k] += sum over a chunk of tokens of da[t][c] q[t][k]; 256 threads,
// 16 outputs each, tokens staged 64 at a time
constexpr int DWG_CHUNK = 4096;
__global__ void __launch_bounds__(256) dwg_kernel(const float* da, const __nv_bfloat16* q, long long tokens,
                                                  float* dwg) {
  __shared__ float sa[64][65];
  __shared__ float sq[64][65];
  const int h = blockIdx.y;
  const long long t0 = static_cast<long long>(blockIdx.x) * DWG_CHUNK;
  const float* dah = da + h * tokens * D;
  const __nv_bfloat16* qh = q + h * tokens * D;
  const int c = threadIdx.x >> 2;                 // output row (channel of da)
  const int k0 = (threadIdx.x & 3) * 16;           // 16 columns
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (long long tb = t0; tb < t0 + DWG_CHUNK && tb < tokens; tb += 64) {
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * 64; e += 256) {
      const int r = e >> 6, cc = e & 63;
      const bool ok = tb + r < tokens;
      sa[r][cc] = ok ? dah[(tb + r) * D + cc] : 0.f;
      sq[r][cc] = ok ? __bfloat162float(qh[(tb + r) * D + cc]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 64; ++r) {
      const float av = sa[r][c];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf(av, sq[r][k0 + i], acc[i]);
    }
  }
  float* out = dwg + static_cast<long long>(h) * D * D + c * D + k0;
#pragma unroll
  for (int i = 0; i < 16; ++i) atomicAdd(out + i, acc[i]);
}

}  // namespace

cudaError_t launch_pool_bwd(const PoolBwdArgs& a, cudaStream_t st) {
  const long long total = static_cast<long long>(a.H) * a.F * a.Hp * a.Wp * (D / 4);
  pool_bwd_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rowdot(const float* do32, const __nv_bfloat16* do16, const float* o32, const __nv_bfloat16* o16,
                          long long rows, float* D_, __nv_bfloat16* do16_out, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  rowdot_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(do32, do16, o32, o16, rows, D_, do16_out);
  return cudaGetLastError();
}

cudaError_t launch_dwg(const float* da, const __nv_bfloat16* q, int H, long long tokens, float* dwg, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(dwg, 0, sizeof(float) * H * D * D, st);
  if (e != cudaSuccess) return e;
  dwg_kernel<<<dim3(static_cast<unsigned>((tokens + DWG_CHUNK - 1) / DWG_CHUNK), H), 256, 0, st>>>(da, q, tokens, dwg);
  return cudaGetLastError();
}

}  // namespace gsa
