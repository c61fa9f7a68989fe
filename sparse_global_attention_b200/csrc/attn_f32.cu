// fp32 attention for fp32 contexts (small configs): one thread per query row,
// fp32 FMA dot products, online softmax with expf.  Serves the compressed
// branch with its streaming top-k (the same exact (score desc, region asc)
// list as the tensor-core kernel, kept in local memory), the special tokens
// and the dense comparison.  "Speed3R: Sparse Feed-forward 3D Reconstruction
// Models" (Paper-Notes, CVPR 2026), compression branch, special-token full
// attention.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

__device__ __forceinline__ bool better(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

template <bool TOPK>
__global__ void __launch_bounds__(64) attn_f32_kernel(const AttnF32Args a) {
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= static_cast<long long>(a.H) * a.n_q) return;
  const int h = static_cast<int>(tid / a.n_q);
  const int row = static_cast<int>(tid - static_cast<long long>(h) * a.n_q);
  const float* q = a.q + h * a.q_hs + static_cast<long long>(row) * D;
  float qr[D], acc[D];
  for (int d = 0; d < D; ++d) { qr[d] = q[d]; acc[d] = 0.f; }
  float lsc[TOPK ? KC_MAX : 1];
  int lid[TOPK ? KC_MAX : 1];
  int lcount = 0;
  float mx = -INFINITY, l = 0.f;
  for (int seg = 0; seg < a.nseg; ++seg) {
    const float* kh = (seg ? a.k[1] : a.k[0]) + h * (seg ? a.kv_hs[1] : a.kv_hs[0]);
    const float* vh = (seg ? a.v[1] : a.v[0]) + h * (seg ? a.kv_hs[1] : a.kv_hs[0]);
    const int nk = seg ? a.n_k[1] : a.n_k[0];
    const int km = seg ? a.kmask[1] : a.kmask[0];
    for (int j = 0; j < nk; ++j) {
      if (!key_valid(km, a.g, j)) continue;
      const float* kp = kh + static_cast<long long>(j) * D;
      float raw = 0.f;
      for (int d = 0; d < D; ++d) raw = fmaf(qr[d], kp[d], raw);
      if constexpr (TOPK) {
        bool cand = true;
        const int fr = j / a.rpf;
        for (int i = 0; i < a.n_fixed; ++i) cand = cand && (a.fixed[i] != fr);
        if (cand && (lcount < a.kc || better(raw, j, lsc[a.kc - 1], lid[a.kc - 1]))) {
          int p = lcount < a.kc ? lcount : a.kc - 1;
          while (p > 0 && better(raw, j, lsc[p - 1], lid[p - 1])) {
            lsc[p] = lsc[p - 1];
            lid[p] = lid[p - 1];
            --p;
          }
          lsc[p] = raw;
          lid[p] = j;
          if (lcount < a.kc) ++lcount;
        }
      }
      const float sc = raw * a.scale;
      const float mn = fmaxf(mx, sc);
      const float al = expf(mx - mn);
      const float pw = expf(sc - mn);
      l = l * al + pw;
      const float* vp = vh + static_cast<long long>(j) * D;
      for (int d = 0; d < D; ++d) acc[d] = acc[d] * al + pw * vp[d];
      mx = mn;
    }
  }
  float inv = l > 0.f ? 1.f / l : 0.f;
  if (a.q_mask != MASK_NONE && !key_valid(a.q_mask, a.g, row)) inv = 0.f;
  float* out = a.o + h * a.o_hs + static_cast<long long>(row) * D;
  for (int d = 0; d < D; ++d) out[d] = acc[d] * inv;
  if constexpr (TOPK) {
    for (int j = 0; j < a.kc; ++j) {
      const int v = j < lcount ? lid[j] : -1;
      a.cand[tid * a.kc + j] = v;
      if (a.cand_user) a.cand_user[tid * a.kc + j] = v;
    }
  }
}

}  // namespace

cudaError_t launch_attn_f32(const AttnF32Args& a, bool topk, cudaStream_t st) {
  const long long n = static_cast<long long>(a.H) * a.n_q;
  const unsigned blocks = static_cast<unsigned>((n + 63) / 64);
  if (topk)
    attn_f32_kernel<true><<<blocks, 64, 0, st>>>(a);
  else
    attn_f32_kernel<false><<<blocks, 64, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gsa
