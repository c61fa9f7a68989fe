// Descriptor tokens of FlashVGGT's descriptor attention.
//
// "FlashVGGT: Efficient and Scalable Visual Geometry Transformers with
// Compressed Descriptor Attention" (Paper-Notes, CVPR 2026), key designs
// "空间压缩描述符Token" and "描述符注意力机制": each frame's (H, W) token grid is
// resized by bilinear interpolation to (H/r, W/r) descriptors, and every
// full-resolution token attends to the descriptors of all frames (plus the
// special tokens) instead of to every token.
//
// Resize convention (the pages name only "bilinear"): output (i, j) of the
// Hd x Wd grid, Hd = floor(Hv / r), samples the valid Hv x Wv grid at
// y = (i + 1/2) * Hv / Hd - 1/2 (clamped below at 0), likewise x, and blends
// the four neighbours (the last row/column repeats at the border).  The
// interpolation is applied to K and V directly: it is linear with weights
// summing to 1, so it commutes with the K/V projections.
//
// One thread makes one 16-byte chunk of one descriptor row: four 16-byte
// loads, fp32 blend, bf16 (round to nearest) or fp32 store.  blockIdx.y picks
// K or V.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* f) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ void store8(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// source index pair and the weight of the second for output i of n_out over n_in
__device__ __forceinline__ void src_of(int i, int n_in, int n_out, int& i0, int& i1, float& w) {
  float y = (static_cast<float>(i) + 0.5f) * (static_cast<float>(n_in) / static_cast<float>(n_out)) - 0.5f;
  y = fmaxf(y, 0.f);
  i0 = min(static_cast<int>(y), n_in - 1);
  i1 = min(i0 + 1, n_in - 1);
  w = y - static_cast<float>(i0);
}

template <typename T>
__global__ void __launch_bounds__(256) desc_kernel(DescArgs a) {
  const int t = blockIdx.y;                       // 0 K, 1 V
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per = a.Hd * a.Wd;
  const long long total = static_cast<long long>(a.H) * a.F * per * (D / 8);
  if (gid >= total) return;
  const int c = static_cast<int>(gid % (D / 8));
  const long long row = gid / (D / 8);            // (h * F + f) * per + i * Wd + j
  const int o = static_cast<int>(row % per);
  const long long hf = row / per;
  const long long hh = hf / a.F, ff = hf - hh * a.F;
  const int i = o / a.Wd, j = o - i * a.Wd;
  int y0, y1, x0, x1;
  float wy, wx;
  src_of(i, a.Hv, a.Hd, y0, y1, wy);
  src_of(j, a.Wv, a.Wd, x0, x1, wx);
  const T* src = reinterpret_cast<const T*>(a.src[t]) + hf * a.Hp * a.Wp * D + c * 8;
  float v00[8], v01[8], v10[8], v11[8], out[8];
  load8(src + (static_cast<long long>(y0) * a.Wp + x0) * D, v00);
  load8(src + (static_cast<long long>(y0) * a.Wp + x1) * D, v01);
  load8(src + (static_cast<long long>(y1) * a.Wp + x0) * D, v10);
  load8(src + (static_cast<long long>(y1) * a.Wp + x1) * D, v11);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float top = v00[e] + wx * (v01[e] - v00[e]);
    const float bot = v10[e] + wx * (v11[e] - v10[e]);
    out[e] = top + wy * (bot - top);
  }
  store8(reinterpret_cast<T*>(a.dst[t]) + hh * a.dst_hs + (ff * per + o) * D + c * 8, out);
}

}  // namespace

cudaError_t launch_descriptors(const DescArgs& a, bool fp32, cudaStream_t st) {
  const long long total = static_cast<long long>(a.H) * a.F * a.Hd * a.Wd * (D / 8);
  dim3 grid(static_cast<unsigned>((total + 255) / 256), 2);
  if (fp32) desc_kernel<float><<<grid, 256, 0, st>>>(a);
  else desc_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gsa
