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
// Kernels (the dense attention backward of the compressed branch and the
// special tokens runs on tcgen05, in attn_tc.cu):
//   sel_bwd     one warp per window: recomputes the selection forward, runs the
//       gate backward, writes dO'_comp of its region and dq of its tokens, and
//       adds dK/dV of its keys (shared by many windows) with fp32 atomics.
//   pool_bwd, dwg_kernel, rowdot  the elementwise and reduction steps.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

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
constexpr int DWG_CHUNK = 4096;                   // tokens per CTA
// dW_g[h] += sum over the CTA's tokens of da[t] q[t]^T: 64-token blocks staged
// in shared memory as fp32, each thread a 4 x 4 tile of the 64 x 64 result
// (two 16-byte shared loads per 16 FMAs), one atomic add per output at the end
__global__ void __launch_bounds__(256) dwg_kernel(const float* da, const __nv_bfloat16* q, long long tokens,
                                                  float* dwg) {
  __shared__ __align__(16) float sa[64][68];       // [token][channel of da]
  __shared__ __align__(16) float sq[64][68];       // [token][channel of q]
  const int h = blockIdx.y;
  const long long t0 = static_cast<long long>(blockIdx.x) * DWG_CHUNK;
  const float* dah = da + h * tokens * D;
  const __nv_bfloat16* qh = q + h * tokens * D;
  const int tc = (threadIdx.x >> 4) * 4;           // rows tc..tc+3 of dW_g (channels of da)
  const int tk = (threadIdx.x & 15) * 4;           // columns tk..tk+3 (channels of q)
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (long long tb = t0; tb < t0 + DWG_CHUNK && tb < tokens; tb += 64) {
    __syncthreads();
#pragma unroll
    for (int it = 0; it < 4; ++it) {                // da: 64 x 64 fp32 as float4
      const int e = threadIdx.x + 256 * it, r = e >> 4, c4 = (e & 15) * 4;
      const bool ok = tb + r < tokens;
      const float4 v = ok ? *reinterpret_cast<const float4*>(dah + (tb + r) * D + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(&sa[r][c4]) = v;
    }
#pragma unroll
    for (int it = 0; it < 2; ++it) {                // q: 64 x 64 bf16 as 8-element pieces
      const int e = threadIdx.x + 256 * it, r = e >> 3, c8 = (e & 7) * 8;
      const bool ok = tb + r < tokens;
      const uint4 raw = ok ? *reinterpret_cast<const uint4*>(qh + (tb + r) * D + c8) : make_uint4(0u, 0u, 0u, 0u);
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw);
      *reinterpret_cast<float4*>(&sq[r][c8]) =
          make_float4(__low2float(b[0]), __high2float(b[0]), __low2float(b[1]), __high2float(b[1]));
      *reinterpret_cast<float4*>(&sq[r][c8 + 4]) =
          make_float4(__low2float(b[2]), __high2float(b[2]), __low2float(b[3]), __high2float(b[3]));
    }
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < 64; ++r) {
      const float4 a = *reinterpret_cast<const float4*>(&sa[r][tc]);
      const float4 b = *reinterpret_cast<const float4*>(&sq[r][tk]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  float* out = dwg + static_cast<long long>(h) * D * D;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) atomicAdd(out + (tc + i) * D + tk + j, acc[i][j]);
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
