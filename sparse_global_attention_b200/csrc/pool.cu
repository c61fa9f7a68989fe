// K1: s x s non-overlapping mean pooling of Q/K/V image tokens.
//
// "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (Paper-Notes,
// CVPR 2026), compression branch: Q_img, K_img, V_img are downsampled by
// s x s non-overlapping average pooling to Q_comp, K_comp, V_comp with
// M'_img = M_img / s^2 rows.  On padded grids the mean runs over the valid
// tokens of each region only.
//
// One thread produces one 16-byte chunk (8 bf16 or 4 fp32 channels) of one
// pooled row: it issues the s*s independent 16-byte loads of its region at
// once (the loop is unrolled for the compile-time s), sums in fp32 and writes
// the mean in bf16 and/or fp32.  For the guide scores the bf16 value also
// gets its residual x - bf16(x) rounded to bf16 (a hi/lo split that carries
// 16 significant bits), so S_guide can be formed on bf16 tensor cores with
// near-fp32 accuracy.  Consecutive threads take consecutive chunks
// of one row, then the next region along x, so each warp reads whole 128-byte
// token rows.  The grid's y dimension selects Q, K or V so one launch pools
// all three tensors.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float* f) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float* f) {
    float4 u = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  }
};

template <typename T, int S>
__global__ void __launch_bounds__(256) pool_kernel(PoolArgs a) {
  constexpr int VN = Vec16<T>::N;
  constexpr int CH = D / VN;                    // chunks per token row
  const int t = blockIdx.y;                     // 0 Q, 1 K, 2 V
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int rpf_x = a.Wp / S;
  const int rpf = (a.Hp / S) * rpf_x;
  const long long total = static_cast<long long>(a.H) * a.F * rpf * CH;
  if (gid >= total) return;
  const int c = static_cast<int>(gid % CH);
  const long long row = gid / CH;               // h * R + r
  const int r_in_f = static_cast<int>(row % rpf);
  const long long hf = row / rpf;               // h * F + f
  const int i = r_in_f / rpf_x;
  const int j = r_in_f - i * rpf_x;
  const void* srcb = t == 0 ? a.src[0] : (t == 1 ? a.src[1] : a.src[2]);
  float* out32 = t == 0 ? a.out32[0] : (t == 1 ? a.out32[1] : a.out32[2]);
  __nv_bfloat16* out16 = t == 0 ? a.out16[0] : (t == 1 ? a.out16[1] : a.out16[2]);
  __nv_bfloat16* outlo = t == 0 ? a.outlo[0] : (t == 1 ? a.outlo[1] : a.outlo[2]);
  const T* src = reinterpret_cast<const T*>(srcb) +
                 ((hf * a.Hp + static_cast<long long>(i) * S) * a.Wp + static_cast<long long>(j) * S) * D +
                 c * VN;
  float acc[VN];
#pragma unroll
  for (int e = 0; e < VN; ++e) acc[e] = 0.f;
  int cnt = 0;
#pragma unroll
  for (int y = 0; y < S; ++y)
#pragma unroll
    for (int x = 0; x < S; ++x) {
      const bool ok = (i * S + y < a.Hv) && (j * S + x < a.Wv);
      if (ok) {
        float v[VN];
        Vec16<T>::load(src + (static_cast<long long>(y) * a.Wp + x) * D, v);
#pragma unroll
        for (int e = 0; e < VN; ++e) acc[e] += v[e];
        ++cnt;
      }
    }
  const float inv = 1.f / static_cast<float>(cnt);
#pragma unroll
  for (int e = 0; e < VN; ++e) acc[e] *= inv;
  const long long o = row * D + c * VN;
  if (out32) {
    float4* p = reinterpret_cast<float4*>(out32 + o);
#pragma unroll
    for (int e = 0; e < VN / 4; ++e) p[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
  }
  if (out16) {
    uint32_t w[VN / 2], wl[VN / 2];
#pragma unroll
    for (int e = 0; e < VN / 2; ++e) {
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      const float2 hf = __bfloat1622float2(hi);
      w[e] = *reinterpret_cast<const uint32_t*>(&hi);
      wl[e] = pack_bf16(acc[2 * e] - hf.x, acc[2 * e + 1] - hf.y);   // exact residual, rounded
    }
    if constexpr (VN == 8) {
      *reinterpret_cast<uint4*>(out16 + o) = make_uint4(w[0], w[1], w[2], w[3]);
      if (outlo) *reinterpret_cast<uint4*>(outlo + o) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    } else {
      *reinterpret_cast<uint2*>(out16 + o) = make_uint2(w[0], w[1]);
      if (outlo) *reinterpret_cast<uint2*>(outlo + o) = make_uint2(wl[0], wl[1]);
    }
  }
}

template <typename T>
static cudaError_t launch_pool_t(const PoolArgs& a, cudaStream_t st) {
  constexpr int CH = D / Vec16<T>::N;
  const long long rpf = static_cast<long long>(a.Hp / a.s) * (a.Wp / a.s);
  const long long total = static_cast<long long>(a.H) * a.F * rpf * CH;
  dim3 grid(static_cast<unsigned>((total + 255) / 256), 3);
  switch (a.s) {
    case 1: pool_kernel<T, 1><<<grid, 256, 0, st>>>(a); break;
    case 2: pool_kernel<T, 2><<<grid, 256, 0, st>>>(a); break;
    case 4: pool_kernel<T, 4><<<grid, 256, 0, st>>>(a); break;
    case 8: pool_kernel<T, 8><<<grid, 256, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_pool(const PoolArgs& a, bool fp32, cudaStream_t st) {
  return fp32 ? launch_pool_t<float>(a, st) : launch_pool_t<__nv_bfloat16>(a, st);
}

}  // namespace gsa
