// Attention core on bf16 tensor cores with fp32 accumulation (flash-style
// online softmax), shared by three steps of the layer:
//   K2  compressed branch: O'_comp = softmax(Q_comp K_comp^T / sqrt(d)) V_comp
//       plus, fused in the same pass, a streaming top-k of the raw guide scores
//       S_guide = Q_comp K_comp^T per compressed query row, so S_guide never
//       leaves the chip ("Speed3R: Sparse Feed-forward 3D Reconstruction
//       Models", Paper-Notes CVPR 2026, compression branch and "高效 Triton
//       Kernel 实现": streaming top-k folded into the FlashAttention loop);
//   K5  special tokens: O_spec = softmax(Q_spec K^T / sqrt(d)) V over every
//       special and valid image token (special-token full attention), split
//       over key ranges and merged by merge_kernel;
//   K6  dense global attention over every token (the comparison baseline).
//
// CTA = 4 warps = 64 query rows; keys stream through shared memory in 64-key
// tiles with a two-stage cp.async pipeline; each warp owns 16 rows and runs
// m16n8k16 MMAs for S = Q K^T and O += P V.
//
// Guide-score precision (K2): Q_comp and K_comp arrive as bf16 pairs
// hi + lo (lo = bf16 of the residual), and S = Qhi Khi^T + Qhi Klo^T +
// Qlo Khi^T.  The dropped Qlo Klo^T term and the split errors are ~2^-17 of
// |q||k|, so the top-k decisions match exact scores far inside the 1e-3
// relative gap that separates a well-defined k-th from the (k+1)-th region.
// The same S feeds the softmax.
//
// Streaming top-k (K2): per row the CTA keeps, in shared memory, the k best
// (score, region) pairs ordered by score descending then region ascending,
// and a threshold T = the k-th score once the list is full.  Per tile, a
// thread whose largest score of a row beats T appends its scores > T of
// candidate regions to the row's small buffer (positions by shared-memory
// atomics); one thread per row then merges the buffer into the list by
// insertion and T is refreshed.  If a buffer would overflow, the entries that
// did not fit are retried against the raised T.  Tiles run in increasing
// region order, so a later score equal to T belongs to a higher region index
// and loses the tie: the strict '>' filter is exact.
#include "gsa_common.cuh"
#include "gsa_kernels.h"

namespace gsa {

namespace {

constexpr int BM = 64;           // query rows per CTA
constexpr int BN = 64;           // keys per tile
constexpr int TILE_BYTES = BN * 128;
constexpr int Q_BYTES = BM * 128;
constexpr int NSTAGE = 2;
constexpr int BUF_CAP = 16;      // top-k append buffer entries per row
constexpr int BUF_ST = BUF_CAP + 1;

template <bool TOPK>
struct Smem {
  static constexpr int NT = TOPK ? 3 : 2;                 // K (hi), [K lo], V tiles per stage
  static constexpr int STAGE = NT * TILE_BYTES;
  static constexpr int Q = TOPK ? 2 * Q_BYTES : Q_BYTES;
  static constexpr int KV = Q;
  static constexpr int LIST = KV + NSTAGE * STAGE;         // byte offset of the top-k area
  static int bytes(int kc) {
    return LIST + (TOPK ? (BM * (kc + 1) * 8 + BM * BUF_ST * 8 + BM * 4) : 0);
  }
};

__device__ __forceinline__ bool better(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

template <bool TOPK>
__device__ __forceinline__ void issue_tile(const AttnArgs& a, int h, int tt, uint32_t stage) {
  const int seg = (a.nseg > 1 && tt >= a.tiles0) ? 1 : 0;
  const int lt = seg ? tt - a.tiles0 : tt;
  const long long kb = static_cast<long long>(lt) * BN;
  const long long hoff = h * a.kv_hs[seg];
  const __nv_bfloat16* kp = a.k[seg] + hoff;
  const __nv_bfloat16* vp = a.v[seg] + hoff;
  const int nk = a.n_k[seg];
#pragma unroll
  for (int it = 0; it < (BN * 8) / 128; ++it) {
    const int e = threadIdx.x + it * 128;
    const int r = e >> 3, c = e & 7;
    const long long key = kb + r;
    const bool ok = key < nk;
    const long long off = (ok ? key : 0) * D + c * 8;
    cp_async16(stage + swz(r, c), kp + off, ok ? 16 : 0);
    cp_async16(stage + (Smem<TOPK>::NT - 1) * TILE_BYTES + swz(r, c), vp + off, ok ? 16 : 0);
    if constexpr (TOPK) cp_async16(stage + TILE_BYTES + swz(r, c), a.k_lo + hoff + off, ok ? 16 : 0);
  }
}

template <bool TOPK>
__global__ void __launch_bounds__(128) attn_kernel(const AttnArgs a) {
  using SM = Smem<TOPK>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + SM::KV;
  const int LST = a.kc + 1;                                   // padded list row stride
  float* lsc = reinterpret_cast<float*>(smem + SM::LIST);     // [BM][LST]
  int* lid = reinterpret_cast<int*>(lsc + BM * LST);
  float* bsc = reinterpret_cast<float*>(lid + BM * LST);      // [BM][BUF_ST]
  int* bid = reinterpret_cast<int*>(bsc + BM * BUF_ST);
  int* bcnt = bid + BM * BUF_ST;                              // [BM]
  if (TOPK && threadIdx.x < BM) bcnt[threadIdx.x] = 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, lr = lane & 7;
  const int h = blockIdx.z, split = blockIdx.y;
  const int row0 = blockIdx.x * BM;
  const float sl2 = a.scale_log2;

  // ---- Q tile (and its low part for the guide scores) -----------------------
  {
    const long long qoff = h * a.q_hs;
#pragma unroll
    for (int it = 0; it < (BM * 8) / 128; ++it) {
      const int e = threadIdx.x + it * 128;
      const int r = e >> 3, c = e & 7;
      const int gr = row0 + r;
      const bool ok = gr < a.n_q;
      const long long off = qoff + static_cast<long long>(ok ? gr : 0) * D + c * 8;
      cp_async16(sQ + swz(r, c), a.q + off, ok ? 16 : 0);
      if constexpr (TOPK) cp_async16(sQ + Q_BYTES + swz(r, c), a.q_lo + off, ok ? 16 : 0);
    }
    cp_async_commit();
  }
  const int t_begin = split * a.tiles_per_split;
  const int t_end = min(t_begin + a.tiles_per_split, a.tiles_total);
  if (t_begin < t_end) issue_tile<TOPK>(a, h, t_begin, sKV);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();

  uint32_t qf[4][4], qlo[TOPK ? 4 : 1][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const uint32_t ad = swz(warp * 16 + lr + 8 * (mi & 1), 2 * ks + (mi >> 1));
    ldsm_x4(sQ + ad, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
    if constexpr (TOPK) ldsm_x4(sQ + Q_BYTES + ad, qlo[ks][0], qlo[ks][1], qlo[ks][2], qlo[ks][3]);
  }

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};
  float thr[2] = {-INFINITY, -INFINITY};
  int lcount = 0;   // list length of row my_row, kept by threads t < 2
  const int my_row = warp * 16 + g + 8 * (t & 1);

  for (int tt = t_begin; tt < t_end; ++tt) {
    const int st = (tt - t_begin) & 1;
    if (tt + 1 < t_end) issue_tile<TOPK>(a, h, tt + 1, sKV + (st ^ 1) * SM::STAGE);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = sKV + st * SM::STAGE;
    const uint32_t sV = sK + (SM::NT - 1) * TILE_BYTES;

    // ---- S = Q K^T ----------------------------------------------------------
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const uint32_t ad = swz(16 * np + lr + 8 * (mi >> 1), 2 * ks + (mi & 1));
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + ad, b0, b1, b2, b3);
        if constexpr (TOPK) {
          uint32_t c0, c1, c2, c3;
          ldsm_x4(sK + TILE_BYTES + ad, c0, c1, c2, c3);
          mma_bf16(s[2 * np], qf[ks], c0, c1);          // Qhi Klo
          mma_bf16(s[2 * np + 1], qf[ks], c2, c3);
          mma_bf16(s[2 * np], qlo[ks], b0, b1);         // Qlo Khi
          mma_bf16(s[2 * np + 1], qlo[ks], b2, b3);
        }
        mma_bf16(s[2 * np], qf[ks], b0, b1);            // Qhi Khi
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }

    // ---- key validity ---------------------------------------------------------
    const int seg = (a.nseg > 1 && tt >= a.tiles0) ? 1 : 0;
    const long long kb = static_cast<long long>(seg ? tt - a.tiles0 : tt) * BN;
    const int nk = a.n_k[seg];
    const int km = a.kmask[seg];
    if (km != MASK_NONE || kb + BN > nk) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const long long key = kb + 8 * nt + 2 * t + e;
          if (key >= nk || !key_valid(km, a.g, key)) {
            s[nt][e] = -INFINITY;
            s[nt][2 + e] = -INFINITY;
          }
        }
    }

    // thread-local row maxima (shared by the top-k filter and the softmax)
    float mxl[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * rr], s[nt][2 * rr + 1]));
      mxl[rr] = mx;
    }

    // ---- streaming top-k of the guide scores ------------------------------------
    if constexpr (TOPK) {
      bool tile_fixed = false;
      for (int i = 0; i < a.n_fixed; ++i) {
        const long long lo = static_cast<long long>(a.fixed[i]) * a.rpf;
        if (lo < kb + BN && lo + a.rpf > kb) tile_fixed = true;
      }
      uint32_t done[2] = {0u, 0u};   // scores of this tile already handed to the list
      bool again = true;
      while (__any_sync(0xffffffffu, again)) {
        bool app = false, over = false;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          if (mxl[rr] > thr[rr]) {           // some score of this thread may enter the list
            const int row = warp * 16 + g + 8 * rr;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float v = s[nt][2 * rr + e];
                const uint32_t bit = 1u << (2 * nt + e);
                if (v > thr[rr] && !(done[rr] & bit)) {
                  const int col = static_cast<int>(kb) + 8 * nt + 2 * t + e;
                  bool ok = true;
                  if (tile_fixed) {
                    const int fr = col / a.rpf;
                    for (int i = 0; i < a.n_fixed; ++i) ok = ok && (a.fixed[i] != fr);
                  }
                  if (!ok) {
                    done[rr] |= bit;
                  } else {
                    const int p = atomicAdd(&bcnt[row], 1);
                    if (p < BUF_CAP) {
                      bsc[row * BUF_ST + p] = v;
                      bid[row * BUF_ST + p] = col;
                      done[rr] |= bit;
                      app = true;
                    } else {
                      over = true;
                    }
                  }
                }
              }
          }
        }
        again = over;
        if (__any_sync(0xffffffffu, app || over)) {
          __syncwarp();
          float newT = -INFINITY;
          if (t < 2) {
            const int row = my_row;
            const int nb = min(bcnt[row], BUF_CAP);
            float* ls = lsc + row * LST;
            int* li = lid + row * LST;
            for (int j = 0; j < nb; ++j) {
              const float sc = bsc[row * BUF_ST + j];
              const int id = bid[row * BUF_ST + j];
              if (lcount == a.kc && !better(sc, id, ls[a.kc - 1], li[a.kc - 1])) continue;
              int p = lcount < a.kc ? lcount : a.kc - 1;
              while (p > 0 && better(sc, id, ls[p - 1], li[p - 1])) {
                ls[p] = ls[p - 1];
                li[p] = li[p - 1];
                --p;
              }
              ls[p] = sc;
              li[p] = id;
              if (lcount < a.kc) ++lcount;
            }
            bcnt[row] = 0;
            if (lcount == a.kc) newT = ls[a.kc - 1];
          }
          __syncwarp();
          const float t0 = __shfl_sync(0xffffffffu, newT, g * 4 + 0);
          const float t1 = __shfl_sync(0xffffffffu, newT, g * 4 + 1);
          thr[0] = t0;
          thr[1] = t1;
        }
      }
    }

    // ---- online softmax ---------------------------------------------------------
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float mx = mxl[rr];
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
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = ex2(fmaf(s[nt][2 * rr], sl2, -mb));
        const float p1 = ex2(fmaf(s[nt][2 * rr + 1], sl2, -mb));
        s[nt][2 * rr] = p0;
        s[nt][2 * rr + 1] = p1;
        l[rr] += p0 + p1;
      }
      m[rr] = m_new;
    }

    // ---- O += P V -----------------------------------------------------------------
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
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
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue -------------------------------------------------------------------
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 1);
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 2);
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = row0 + warp * 16 + g + 8 * rr;
    if (row >= a.n_q) continue;
    if (a.n_split == 1) {
      float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
      if (a.q_mask != MASK_NONE && !key_valid(a.q_mask, a.g, row)) inv = 0.f;
      const long long base = h * a.o_hs + static_cast<long long>(row) * D;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int d = 8 * nt + 2 * t;
        const float v0 = o[nt][2 * rr] * inv, v1 = o[nt][2 * rr + 1] * inv;
        if (a.o16)
          *reinterpret_cast<uint32_t*>(a.o16 + base + d) = pack_bf16(v0, v1);
        else
          *reinterpret_cast<float2*>(a.o32 + base + d) = make_float2(v0, v1);
      }
    } else {
      const long long pr = (static_cast<long long>(split) * a.H + h) * a.n_q + row;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        *reinterpret_cast<float2*>(a.part_o + pr * D + 8 * nt + 2 * t) =
            make_float2(o[nt][2 * rr], o[nt][2 * rr + 1]);
      if (t == 0) *reinterpret_cast<float2*>(a.part_ml + pr * 2) = make_float2(m[rr], l[rr]);
    }
  }

  if constexpr (TOPK) {
    if (t < 2) {
      const int row = row0 + my_row;
      if (row < a.n_q) {
        const long long base = (static_cast<long long>(h) * a.n_q + row) * a.kc;
        for (int j = 0; j < a.kc; ++j) {
          const int v = (j < lcount) ? lid[my_row * LST + j] : -1;
          a.cand[base + j] = v;
          if (a.cand_user) a.cand_user[base + j] = v;
        }
      }
    }
  }
}

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
}

}  // namespace

cudaError_t launch_attn(const AttnArgs& a, bool topk, cudaStream_t st) {
  dim3 grid((a.n_q + BM - 1) / BM, a.n_split, a.H);
  cudaError_t e;
  if (topk) {
    const int sm = Smem<true>::bytes(a.kc);
    e = cudaFuncSetAttribute(attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    attn_kernel<true><<<grid, 128, sm, st>>>(a);
  } else {
    const int sm = Smem<false>::bytes(0);
    e = cudaFuncSetAttribute(attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    attn_kernel<false><<<grid, 128, sm, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  const long long warps = static_cast<long long>(a.H) * a.n_q;
  merge_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gsa
