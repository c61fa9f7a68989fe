// K4: nearest-neighbour upsample of O'_comp, gate, blend.
//
// "Speed3R: Sparse Feed-forward 3D Reconstruction Models" (Paper-Notes,
// CVPR 2026): compression branch, O_comp = Upsample(O'_comp) by nearest
// neighbour; gated aggregation, g = sigmoid(W_g Q_img) and
// O_img = g * O_comp + (1 - g) * O_sel, with W_g a learned per-head d x d
// projection (row = output channel, no bias) and g per channel.
//
// bf16 path: each warp takes 16 consecutive image tokens; G = Q W_g^T runs as
// m16n8k16 MMAs with W_g staged once per CTA in swizzled shared memory; the
// MMA result fragment tells each thread which (token, channel) pairs it owns,
// and it reads O'_comp (fp32, by the token's region) and O_sel at exactly
// those positions, blends and stores.  CTAs loop over token tiles so W_g is
// loaded once per CTA.  Pad tokens write 0.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

constexpr int EPI_WARPS = 8;
constexpr int EPI_TILES_PER_CTA = 16;   // 16-token tiles per warp and CTA pass

__device__ __forceinline__ float sigmoid_fast(float x) {
  const float e = ex2(fminf(-x * LOG2E, 126.f));
  return __fdividef(1.f, 1.f + e);
}

__device__ __forceinline__ int region_of(const EpiArgs& a, long long n, bool& valid) {
  const int per = a.g.Hp * a.g.Wp;
  const int f = static_cast<int>(n / per);
  const int o = static_cast<int>(n - static_cast<long long>(f) * per);
  const int y = o / a.g.Wp, x = o - y * a.g.Wp;
  valid = y < a.g.Hv && x < a.g.Wv;
  return f * a.rpf + (y / a.s) * (a.g.Wp / a.s) + x / a.s;
}

__global__ void __launch_bounds__(EPI_WARPS * 32) epi_kernel_bf16(const EpiArgs a) {
  __shared__ __align__(128) uint8_t sW[64 * 128];
  __shared__ __align__(128) uint8_t sQall[EPI_WARPS][16 * 128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, lr = lane & 7;
  const int h = blockIdx.y;
  const long long per_head = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
  const long long img_hs = per_head * D;
  const __nv_bfloat16* wg = reinterpret_cast<const __nv_bfloat16*>(a.w_g) + static_cast<long long>(h) * D * D;
  const uint32_t sWa = smem_u32(sW);
  for (int e = threadIdx.x; e < 64 * 8; e += blockDim.x) {
    const int r = e >> 3, c = e & 7;
    cp_async16(sWa + swz(r, c), wg + r * D + c * 8, 16);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  const __nv_bfloat16* qh = reinterpret_cast<const __nv_bfloat16*>(a.q_img) + h * img_hs;
  const __nv_bfloat16* sh = a.o_sel ? reinterpret_cast<const __nv_bfloat16*>(a.o_sel) + h * img_hs : nullptr;
  const float* ch = a.o_comp + static_cast<long long>(h) * a.R * D;
  __nv_bfloat16* oh = reinterpret_cast<__nv_bfloat16*>(a.o_img) + h * img_hs;
  const uint32_t sQ = smem_u32(sQall[warp]);
  const long long ntile = (per_head + 15) / 16;

  for (long long tile = (static_cast<long long>(blockIdx.x) * EPI_WARPS + warp); tile < ntile;
       tile += static_cast<long long>(gridDim.x) * EPI_WARPS) {
    const long long t0 = tile * 16;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = lane + 32 * it;
      const int r = e >> 3, c = e & 7;
      const bool ok = t0 + r < per_head;
      cp_async16(sQ + swz(r, c), qh + (ok ? t0 + r : 0) * D + c * 8, ok ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    float gacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) gacc[i][0] = gacc[i][1] = gacc[i][2] = gacc[i][3] = 0.f;
    if (a.gate_mode == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t qa[4];
        ldsm_x4(sQ + swz(lr + 8 * (mi & 1), 2 * ks + (mi >> 1)), qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sWa + swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1)), b0, b1, b2, b3);
          mma_bf16(gacc[2 * np], qa, b0, b1);
          mma_bf16(gacc[2 * np + 1], qa, b2, b3);
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const long long n = t0 + g + 8 * rr;
      if (n >= per_head) continue;
      bool valid;
      const int reg = region_of(a, n, valid);
      const float* cp = ch + static_cast<long long>(reg) * D;
      const __nv_bfloat16* sp = sh + n * D;
      __nv_bfloat16* op = oh + n * D;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = 8 * nt + 2 * t;
        float out0 = 0.f, out1 = 0.f;
        if (valid) {
          float g0, g1;
          if (a.gate_mode == 1) { g0 = g1 = 1.f; }
          else if (a.gate_mode == 2) { g0 = g1 = 0.f; }
          else { g0 = sigmoid_fast(gacc[nt][2 * rr]); g1 = sigmoid_fast(gacc[nt][2 * rr + 1]); }
          // a forced gate never reads the branch it drops (it may not have been computed)
          const float2 oc = a.gate_mode == 2 ? make_float2(0.f, 0.f) : __ldg(reinterpret_cast<const float2*>(cp + c));
          const float2 os = a.gate_mode == 1 ? make_float2(0.f, 0.f)
                                             : __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sp + c));
          out0 = g0 * oc.x + (1.f - g0) * os.x;
          out1 = g1 * oc.y + (1.f - g1) * os.y;
        }
        *reinterpret_cast<uint32_t*>(op + c) = pack_bf16(out0, out1);
      }
    }
  }
}

// fp32: one thread per (token, channel)
__global__ void __launch_bounds__(256) epi_kernel_f32(const EpiArgs a) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long per_head = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
  if (tid >= per_head * a.H * D) return;
  const int c = static_cast<int>(tid % D);
  const long long hn = tid / D;
  const int h = static_cast<int>(hn / per_head);
  const long long n = hn - h * per_head;
  bool valid;
  const int reg = region_of(a, n, valid);
  float* out = reinterpret_cast<float*>(a.o_img) + hn * D + c;
  if (!valid) { *out = 0.f; return; }
  const float* q = reinterpret_cast<const float*>(a.q_img) + hn * D;
  const float* w = reinterpret_cast<const float*>(a.w_g) + (static_cast<long long>(h) * D + c) * D;
  float gsum = 0.f;
  for (int i = 0; i < D; ++i) gsum = fmaf(w[i], q[i], gsum);
  float gv = 1.f / (1.f + expf(-gsum));
  if (a.gate_mode == 1) gv = 1.f;
  if (a.gate_mode == 2) gv = 0.f;
  // a forced gate never reads the branch it drops (it may not have been computed)
  const float oc = a.gate_mode == 2 ? 0.f : a.o_comp[(static_cast<long long>(h) * a.R + reg) * D + c];
  const float os = a.gate_mode == 1 ? 0.f : reinterpret_cast<const float*>(a.o_sel)[hn * D + c];
  *out = gv * oc + (1.f - gv) * os;
}

}  // namespace

cudaError_t launch_epilogue(const EpiArgs& a, bool fp32, cudaStream_t st) {
  const long long per_head = static_cast<long long>(a.F) * a.g.Hp * a.g.Wp;
  if (fp32) {
    const long long n = per_head * a.H * D;
    epi_kernel_f32<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a);
  } else {
    const long long ntile = (per_head + 15) / 16;
    const long long per_cta = static_cast<long long>(EPI_WARPS) * EPI_TILES_PER_CTA;
    dim3 grid(static_cast<unsigned>((ntile + per_cta - 1) / per_cta), a.H);
    epi_kernel_bf16<<<grid, EPI_WARPS * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace gsa
