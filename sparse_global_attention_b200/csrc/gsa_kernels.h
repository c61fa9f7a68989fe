// Host-side launch interface of the GSA kernels (internal to the library).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gsa_common.cuh"

namespace gsa {

// ---- K1 pool ---------------------------------------------------------------
struct PoolArgs {
  const void* src[3];        // Q/K/V image tokens [H][F][Hp][Wp][64]
  __nv_bfloat16* out16[3];   // pooled, bf16 (round to nearest) [H][R][64]  (nullptr = skip)
  __nv_bfloat16* outlo[3];   // pooled minus its bf16 value, in bf16         (nullptr = skip)
  float* out32[3];           // pooled, fp32 [H][R][64]                      (nullptr = skip)
  int H, F, Hp, Wp, Hv, Wv, s;
};
cudaError_t launch_pool(const PoolArgs& a, bool fp32, cudaStream_t st);

// ---- FlashVGGT descriptors: bilinear resize of K/V to (Hv/r, Wv/r) per frame --
struct DescArgs {
  const void* src[2];        // K, V image tokens [H][F][Hp][Wp][64]
  void* dst[2];              // descriptors [H][F][Hd][Wd][64] (head stride dst_hs), context dtype
  long long dst_hs;          // elements per head in dst
  int H, F, Hp, Wp, Hv, Wv, Hd, Wd;
};
cudaError_t launch_descriptors(const DescArgs& a, bool fp32, cudaStream_t st);

// ---- attention core (K2 compressed + top-k, K5 special, K6 dense) ----------
struct AttnArgs {
  const __nv_bfloat16* q;    // [H][n_q][64]
  const __nv_bfloat16* q_lo; // top-k only: low bf16 parts of q and k[0]
  const __nv_bfloat16* k_lo;
  long long q_hs;            // head stride (elements)
  int n_q;                   // query rows per head
  int q_mask;                // MASK_NONE or MASK_DENSE: pad query rows output 0
  int nseg;                  // 1 or 2 key segments, tiled separately
  const __nv_bfloat16* k[2];
  const __nv_bfloat16* v[2];
  long long kv_hs[2];
  int n_k[2];
  int kmask[2];              // MaskMode per segment
  // optional per segment: key validity bits (bit e of word w = key 32 w + e of a
  // head, zero from n_k up to the next 128-key tile), used instead of kmask
  // (launches without the top-k)
  const uint32_t* kbits[2];
  int guide_only;            // top-k only: S and the top-k, no P V and no output
  float* lse;                // optional [H][n_q] base-2 log-sum-exp per row (n_split == 1)
  int tiles0;                // 128-key tiles of segment 0
  int tiles_total;
  int tiles_per_split;
  int n_split;               // 1 = write final output, >1 = write partials
  int H;
  Grid g;
  float scale_log2;          // softmax scale * log2(e)
  __nv_bfloat16* o16;        // final output [H][n_q][64] (one of o16/o32)
  float* o32;
  long long o_hs;
  float* part_o;             // [n_split][H][n_q][64] unnormalised
  float* part_ml;            // [n_split][H][n_q][2]  (running max in raw score units, sum)
  // streaming top-k of the raw scores (compressed branch only)
  int kc;                    // regions kept per row by this launch (<= 32)
  int* cand;                 // [H][n_q][kc] region indices, best first (with several passes:
  int* cand_user;            //   [H][n_q][cand_stride], this launch's from column cand_off);
                             //   cand_user: optional copy
  int rpf;                   // regions per frame
  int n_fixed;
  int fixed[MAX_FIXED];      // frames excluded from the candidates
  int* err;                  // device error word
  // top-k in several passes of at most 32: every pass writes its last entry per row
  // to last_s / last_i; a pass after the first (guide only) continues the selection
  // after the previous pass's last entry (excl_s score, excl_i region)
  int cand_stride, cand_off;
  const float* excl_s;
  const int* excl_i;
  float* last_s;
  int* last_i;
};
// tcgen05/TMEM/TMA version: 2 x 128 query rows per CTA, 128-key tiles; the
// top-k runs when a.kc > 0 (a.q_lo / a.k_lo required)
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st);
int attn_tc_tiles(long long n);
// key-range splits for a launch of n_q query rows per head over tiles_total
// 128-key tiles (rows of every split are merged by launch_merge)
void attn_tc_split(int H, long long n_q, int tiles_total, int* tiles_per_split, int* n_split);

struct MergeArgs {
  const float* part_o;
  const float* part_ml;
  int n_split, H, n_q;
  float scale_log2;
  __nv_bfloat16* o16;
  float* o32;
  long long o_hs;
  float* lse;                // optional [H][n_q] base-2 log-sum-exp of each row (backward)
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st);

// ---- K3 selection ----------------------------------------------------------
struct SelArgs {
  const void* q_img;         // [H][F][Hp][Wp][64]
  const void* k_img;
  const void* v_img;
  const void* k_spec;        // [H][F][ns][64]
  const void* v_spec;
  const int* idx;            // [H][R][topk]
  void* o_sel;               // [H][F][Hp][Wp][64]
  int H, F, R, rpf, topk, s;
  Grid g;
  float scale_log2;
  int n_fixed;
  int fixed[MAX_FIXED];
  // optional (bf16 fused kernel): the fixed context's attention computed apart, as
  // the normalised output [H][F*Hp*Wp][64] fp32 and its base-2 log-sum-exp
  // [H][F*Hp*Wp]; the selection then attends only the dynamic keys and merges
  const float* fix_o;
  const float* fix_lse;
  int* err;
};
cudaError_t launch_sel(const SelArgs& a, bool fp32, cudaStream_t st);
// the fixed frames' valid keys and values, packed per head as [H][n_fixed * (ns + Hv*Wv)][64]
// (per fixed frame its special tokens, then its valid image tokens row-major)
cudaError_t launch_fixed_gather(const SelArgs& a, __nv_bfloat16* kfix, __nv_bfloat16* vfix, cudaStream_t st);

// ---- K3 + K4 on tcgen05 (bf16, s = 4): groups of SEL_GROUP neighbouring windows
// (8 x 16 queries = one 128-row MMA tile) attend to the union of their selected
// regions, each row masked to its own window's regions --------------------------
constexpr int SEL_GROUP = 8;
constexpr int SEL_UNION_MAX = 1024;          // SEL_GROUP * top-k <= this (top-k <= 128)
struct SelTcArgs {
  const void* q_img;         // [H][F][Hp][Wp][64] bf16
  const void* k_img;
  const void* v_img;
  const void* w_g;           // [H][64][64] bf16 (gate_mode 0)
  const int* idx;            // [H][R][topk] selected regions
  const int* win_of;         // [R] window at each group position (sel_group_order)
  const int* grp_of;         // [NG] groups in processing order (sel_group_schedule)
  uint2* uni;                // [H][NG][emax] union entries: x region, y = (token bits << 16) | window bits
  int* ucnt;                 // [H][NG] distinct regions per group
  int emax;                  // SEL_GROUP * topk
  int NG;                    // groups per head
  int topk;
  const float* o_comp;       // O'_comp [H][R][64] fp32
  const float* fix_o;        // optional fixed-context attention [H][F*Hp*Wp][64] fp32 and its
  const float* fix_lse;      //   base-2 log-sum-exp [H][F*Hp*Wp]
  __nv_bfloat16* o_img;      // [H][F][Hp][Wp][64]
  __nv_bfloat16* o_sel;      // optional [H][F][Hp][Wp][64]
  int H, F, R, rpf, rx;      // rx = Wp / 4 windows per region row
  Grid g;
  float scale_log2;
  int gate_mode;             // 0 g = sigmoid(W_g q), 1 g = 1, 2 g = 0
  int* err;
};
int sel_group_count(int R);
// group positions -> windows: per frame, row pairs top to bottom, walking the
// columns alternately left to right and back (win_of has F * rows * cols entries)
void sel_group_order(int F, int rows, int cols, int* win_of);
// processing order of a head's groups: by the groups' position inside their frame
// first, frame second, so that the groups in flight at once sit at the same place in
// many frames and select overlapping regions (their K/V stays in L2)
void sel_group_schedule(int F, int rpf, int NG, int* grp_of);
cudaError_t launch_sel_union(const SelTcArgs& a, cudaStream_t st);
cudaError_t launch_sel_tc(const SelTcArgs& a, cudaStream_t st);

// ---- K4 upsample + gate + blend --------------------------------------------
struct EpiArgs {
  const void* q_img;         // [H][F][Hp][Wp][64]
  const void* o_sel;         // [H][F][Hp][Wp][64]
  const float* o_comp;       // [H][R][64] fp32
  const void* w_g;           // [H][64][64]
  void* o_img;               // [H][F][Hp][Wp][64]
  int H, F, R, rpf, s;
  Grid g;
  int gate_mode;
};
cudaError_t launch_epilogue(const EpiArgs& a, bool fp32, cudaStream_t st);

// ---- K3 + K4 fused (bf16, s in {1, 2, 4}): selection attention, then the
// upsample/gate/blend of the window's tokens in the same kernel -------------
cudaError_t launch_sel_fused(const SelArgs& a, const EpiArgs& ep, cudaStream_t st);

// ---- fp32 (SIMT) variants for fp32 contexts ---------------------------------
struct AttnF32Args {
  const float* q; long long q_hs; int n_q; int q_mask;
  int nseg;
  const float* k[2]; const float* v[2]; long long kv_hs[2]; int n_k[2]; int kmask[2];
  int H; Grid g; float scale;
  float* o; long long o_hs;
  int kc; int* cand; int* cand_user; int rpf; int n_fixed; int fixed[MAX_FIXED];
};
cudaError_t launch_attn_f32(const AttnF32Args& a, bool topk, cudaStream_t st);

// ---- allocation-free calls: their device status word (static device memory) --
int noalloc_status_word(int** out);

// ---- failure-detection self-test ---------------------------------------------
// one CTA waits on an mbarrier that nothing completes, gives up after limit_ns
// of global time and records the timeout code in *err
cudaError_t launch_expire_wait(int* err, unsigned long long limit_ns, cudaStream_t st);

// ---- backward ----------------------------------------------------------------
// dense attention backward (flash style) for one query set against up to two
// key segments; P is recomputed from the forward's base-2 log-sum-exp
struct BwdArgs {
  const __nv_bfloat16* q;    // [H][n_q][64]
  const __nv_bfloat16* q_lo; // optional low parts of q and k[0] (split scores), else nullptr
  const __nv_bfloat16* k_lo;
  long long q_hs;
  int n_q;
  int nseg;
  const __nv_bfloat16* k[2];
  const __nv_bfloat16* v[2];
  long long kv_hs[2];
  int n_k[2];
  int kmask[2];
  const __nv_bfloat16* dO;   // [H][n_q][64]
  long long do_hs;
  const float* lse2;         // [H][n_q] log2 sum exp2(S * scale_log2)
  const float* Dv;           // [H][n_q] rowsum(dO o O)
  float* dq;                 // [H][n_q][64] fp32
  long long dq_hs;
  int dq_accum;              // 1: add to dq, 0: overwrite
  float* dk[2];              // [H][n_k][64] fp32 per segment (nullptr: skip the segment)
  float* dv[2];
  long long dkv_hs[2];
  int dkv_accum;
  int H;
  Grid g;
  float scale_log2, scale;
  const uint32_t* kbits[2];  // optional per-segment key validity, 4 words per 128-key tile (as the forward's)
};
// dQ on tcgen05/TMEM/TMA: 128 query rows per CTA; heads packed (q_hs = n_q * 64,
// kv_hs = n_k * 64); split scores (q_lo, k_lo) with one key segment only
cudaError_t launch_attn_bwd_dq_tc(const BwdArgs& a, int* err, cudaStream_t st);
// dK/dV on tcgen05: 128 keys per CTA, one launch per key segment (same layout rules)
cudaError_t launch_attn_bwd_dkv_tc(const BwdArgs& a, int* err, cudaStream_t st);

// selection + gate backward: one warp per window (s <= 4)
struct SelBwdArgs {
  SelArgs s;                 // the forward's selection arguments (o_sel unused)
  const void* w_g;
  const float* o_comp;       // O'_comp [H][R][64]
  const __nv_bfloat16* d_o;  // dO_img [H][F][Hp][Wp][64]
  int gate_mode;
  float* dq;                 // fp32 [H][F][Hp][Wp][64]: written (window tokens)
  float* dk;                 // fp32 image-token dK/dV: atomically added
  float* dv;
  float* dk_spec;            // fp32 [H][F][ns][64] (fixed-frame special keys): atomically added
  float* dv_spec;
  float* d_ocomp;            // fp32 [H][R][64]: written
  float* da;                 // fp32 [H][F][Hp][Wp][64]: gate pre-activation gradient (0 on pads)
  // fixed context computed apart (s.fix_o / s.fix_lse set, bf16): the kernel loops
  // only the selected regions, with P normalised over the union of both key sets,
  // and writes per image token what the dense backward over the fixed keys needs:
  // dO_sel (bf16, 0 on pads), the union's base-2 log-sum-exp (+inf on pads) and
  // D = dO_sel . O_sel
  __nv_bfloat16* dosel;      // [H][F*Hp*Wp][64]
  float* lse_u;              // [H][F*Hp*Wp]
  float* Dq;                 // [H][F*Hp*Wp]
};
cudaError_t launch_sel_bwd(const SelBwdArgs& a, cudaStream_t st);
// gradients of the packed fixed-context keys/values ([H][n_fixed * (ns + Hv*Wv)][64]
// fp32, the layout of launch_fixed_gather) added to the fixed frames' special and
// image tokens
cudaError_t launch_fixed_scatter_add(const SelArgs& a, const float* dkfix, const float* dvfix, float* dk_img,
                                     float* dv_img, float* dk_spec, float* dv_spec, cudaStream_t st);

// pool backward and small steps
struct PoolBwdArgs {
  const float* dcomp[3];     // dQ_comp, dK_comp, dV_comp [H][R][64]
  float* dimg[3];            // += into [H][F][Hp][Wp][64]
  int H, F, Hp, Wp, Hv, Wv, s;
};
cudaError_t launch_pool_bwd(const PoolBwdArgs& a, cudaStream_t st);
// D[h][i] = sum_c dO[h][i][c] * O[h][i][c]; dO fp32 or bf16 (do32 / do16), O fp32 or bf16;
// optional bf16 copy of a fp32 dO
cudaError_t launch_rowdot(const float* do32, const __nv_bfloat16* do16, const float* o32, const __nv_bfloat16* o16,
                          long long rows, float* D, __nv_bfloat16* do16_out, cudaStream_t st);
// dW_g[h] = sum over tokens of da (x) q  ([H][64][64], fp32, overwritten)
cudaError_t launch_dwg(const float* da, const __nv_bfloat16* q, int H, long long tokens, float* dwg, cudaStream_t st);

}  // namespace gsa
