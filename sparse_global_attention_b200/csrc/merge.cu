// Merge of split-key attention partials (K5, special tokens over every token,
// and the special-token queries of the descriptor attention): each split wrote
// per row its running max m_j (raw score units), sum l_j and unnormalised
// output O_j; the row's result is sum_j w_j O_j / sum_j w_j l_j with
// w_j = 2^((m_j - max_j m_j) * scale * log2 e).  One warp per row, two
// channels per lane.  Optionally writes the row's base-2 log-sum-exp
// (max * scale * log2 e + log2 sum) for the backward pass.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.H * a.n_q) return;
  const int h = warp / a.n_q, row = warp - h * a.n_q;
  float mx = -INFINITY;
  for (int j = 0; j < a.n_split; ++j)
    mx = fmaxf(mx, a.part_ml[((static_cast<long long>(j) * a.H + h) * a.n_q + row) * 2]);
  const float mu = (mx == -INFINITY) ? 0.f : mx;
  float l = 0.f, o0 = 0.f, o1 = 0.f;
  for (int j = 0; j < a.n_split; ++j) {
    const long long pr = (static_cast<long long>(j) * a.H + h) * a.n_q + row;
    const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + pr * 2);
    const float w = ex2((ml.x - mu) * a.scale_log2);
    l += w * ml.y;
    const float2 ov = *reinterpret_cast<const float2*>(a.part_o + pr * D + 2 * lane);
    o0 += w * ov.x;
    o1 += w * ov.y;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const long long base = h * a.o_hs + static_cast<long long>(row) * D + 2 * lane;
  if (a.o16)
    *reinterpret_cast<uint32_t*>(a.o16 + base) = pack_bf16(o0 * inv, o1 * inv);
  else
    *reinterpret_cast<float2*>(a.o32 + base) = make_float2(o0 * inv, o1 * inv);
  if (a.lse && lane == 0)
    a.lse[static_cast<long long>(h) * a.n_q + row] = l > 0.f ? mu * a.scale_log2 + __log2f(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  const long long warps = static_cast<long long>(a.H) * a.n_q;
  merge_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gsa
