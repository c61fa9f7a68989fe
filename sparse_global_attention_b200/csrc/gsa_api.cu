// C ABI of the GSA layer: config validation, workspace ownership, kernel
// sequencing on the caller's stream.  See include/gsa.h for the contract.
#include <vector>
#include <math.h>
#include <new>
#include <string.h>

#include "../../include/gsa.h"
#include "gsa_kernels.h"

using namespace gsa;

namespace {

constexpr size_t ALIGN = 256;
constexpr int MAX_EVENTS = 16;
constexpr int MAX_CHUNKS = 16;         // head chunks of the host-buffer pipeline

size_t align_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

struct Derived {
  int rpf, R, ncand, kc;
  long long img_per_head, spec_per_head;
  bool fp32, pads;
  size_t esize;
  int spec_tiles0, spec_tiles_total, spec_split, spec_tps;
};

int validate(const gsa_config* c, Derived* d) {
  if (!c) return GSA_ERR_INVALID_ARG;
  if (c->num_frames < 1 || c->grid_h < 1 || c->grid_w < 1 || c->num_heads < 1 ||
      c->num_special < 0 || c->pool_s < 1 || c->topk < 1)
    return GSA_ERR_INVALID_ARG;
  if (c->dtype != GSA_BF16 && c->dtype != GSA_FP32) return GSA_ERR_INVALID_ARG;
  if (c->gate_mode < 0 || c->gate_mode > 2) return GSA_ERR_INVALID_ARG;
  if (c->num_fixed_frames < 0 || (c->num_fixed_frames > 0 && !c->fixed_frames))
    return GSA_ERR_INVALID_ARG;
  if (c->num_fixed_frames > GSA_MAX_FIXED_FRAMES) return GSA_ERR_UNSUPPORTED;
  if (c->variant < GSA_VARIANT_FULL || c->variant > GSA_VARIANT_DESCRIPTOR) return GSA_ERR_INVALID_ARG;
  if (c->variant == GSA_VARIANT_DESCRIPTOR && (c->grid_h < c->pool_s || c->grid_w < c->pool_s)) return GSA_ERR_SHAPE;
  if (!(c->softmax_scale >= 0.f) || isinf(c->softmax_scale)) return GSA_ERR_INVALID_ARG;
  if (c->head_dim != 64) return GSA_ERR_SHAPE;
  const int s = c->pool_s;
  if (s != 1 && s != 2 && s != 4 && s != 8) return GSA_ERR_UNSUPPORTED;
  if (c->pad_h < c->grid_h || c->pad_w < c->grid_w) return GSA_ERR_SHAPE;
  if (c->pad_h % s || c->pad_w % s) return GSA_ERR_SHAPE;
  // every region needs a valid token: the last region row/col must reach the grid
  if (c->pad_h - s >= c->grid_h || c->pad_w - s >= c->grid_w) return GSA_ERR_SHAPE;
  for (int i = 0; i < c->num_fixed_frames; ++i) {
    const int f = c->fixed_frames[i];
    if (f < 0 || f >= c->num_frames) return GSA_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (c->fixed_frames[j] == f) return GSA_ERR_INVALID_ARG;
  }
  d->rpf = (c->pad_h / s) * (c->pad_w / s);
  const long long R = static_cast<long long>(c->num_frames) * d->rpf;
  d->img_per_head = static_cast<long long>(c->num_frames) * c->pad_h * c->pad_w;
  d->spec_per_head = static_cast<long long>(c->num_frames) * c->num_special;
  if (R * c->num_heads >= (1LL << 31) || d->img_per_head >= (1LL << 31) ||
      d->img_per_head * c->num_heads >= (1LL << 40))
    return GSA_ERR_UNSUPPORTED;
  d->R = static_cast<int>(R);
  d->ncand = d->R - c->num_fixed_frames * d->rpf;
  if (c->topk > d->ncand) return GSA_ERR_SHAPE;
  if (c->topk > GSA_MAX_TOPK) return GSA_ERR_UNSUPPORTED;
  // beyond 64 regions only the bf16 tensor-core selection (4 x 4 windows) takes the list
  if (c->topk > 64 && (c->dtype != GSA_BF16 || s != 4)) return GSA_ERR_UNSUPPORTED;
  d->kc = c->topk;
  d->fp32 = c->dtype == GSA_FP32;
  d->pads = c->pad_h != c->grid_h || c->pad_w != c->grid_w;
  d->esize = d->fp32 ? 4 : 2;
  // special tokens: split the key range so that enough CTAs run
  const long long M = d->spec_per_head;
  d->spec_tiles0 = attn_tc_tiles(M);                                       // 128-key tiles
  d->spec_tiles_total = d->spec_tiles0 + attn_tc_tiles(d->img_per_head);
  attn_tc_split(c->num_heads, M, d->spec_tiles_total, &d->spec_tps, &d->spec_split);
  return GSA_OK;
}

struct Layout {
  size_t comp16[3], complo[2], comp32[3], ocomp, idx, osel, part_o, part_ml, lse_c, lse_s, err, total;
  size_t last_s, last_i;
  // bf16 with fixed frames: the fixed context's keys/values packed per head, and
  // the image queries' attention over them (output, base-2 LSE)
  size_t kfix, vfix, ofix, lsefix;
  long long nfix;   // fixed-context keys per head (0: none)
  // bf16 on a padded grid: validity bits of one head's image tokens (pad slots
  // 0), whole 128-key tiles, written once at create
  size_t kbits;
  size_t kbits_words;
  // the same for the dense layout of gsa_dense_forward (per frame: special tokens, then the grid)
  size_t kbits_dense;
  size_t kbits_dense_words;
  // bf16 selection on tensor cores (s = 4): window order of the groups (written
  // once at create), and per forward the union of each group's selected regions
  size_t winof, grpof, uni, ucnt;
  int ngroups;
};

// the tensor-core selection serves bf16 contexts with 4 x 4 windows that have a selection branch
bool sel_on_tc(const gsa_config* c, const Derived& d) {
  const bool sel = c->variant == GSA_VARIANT_FULL || c->variant == GSA_VARIANT_NO_COMP_VALUE;
  return sel && !d.fp32 && c->pool_s == 4 && c->topk * SEL_GROUP <= SEL_UNION_MAX;
}

Layout make_layout(const gsa_config* c, const Derived& d) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  const size_t rows = static_cast<size_t>(c->num_heads) * d.R;
  for (int i = 0; i < 3; ++i) L.comp16[i] = d.fp32 ? SIZE_MAX : take(rows * D * 2);
  for (int i = 0; i < 2; ++i) L.complo[i] = d.fp32 ? SIZE_MAX : take(rows * D * 2);
  for (int i = 0; i < 3; ++i) L.comp32[i] = d.fp32 ? take(rows * D * 4) : SIZE_MAX;
  L.ocomp = take(rows * D * 4);
  L.idx = take(rows * c->topk * 4);
  L.osel = take(static_cast<size_t>(c->num_heads) * d.img_per_head * D * d.esize);
  const size_t sp = static_cast<size_t>(d.spec_split > 1 ? d.spec_split : 0) * c->num_heads * d.spec_per_head;
  L.part_o = take(sp * D * 4);
  L.part_ml = take(sp * 2 * 4);
  L.lse_c = take(rows * 4);                                                  // for the backward
  // top-k beyond one 32-entry list: each row's last selection of a pass, where the next pass continues
  const bool multi = !d.fp32 && c->topk > 32;
  L.last_s = multi ? take(rows * 4) : SIZE_MAX;
  L.last_i = multi ? take(rows * 4) : SIZE_MAX;
  L.lse_s = take(static_cast<size_t>(c->num_heads) * d.spec_per_head * 4);
  L.err = take(16);
  const bool sel = c->variant != GSA_VARIANT_NO_SELECTION && c->variant != GSA_VARIANT_DESCRIPTOR;
  L.nfix = (!d.fp32 && sel) ? static_cast<long long>(c->num_fixed_frames) * (c->num_special + c->grid_h * c->grid_w) : 0;
  const size_t qrows = static_cast<size_t>(c->num_heads) * d.img_per_head;
  L.kfix = L.nfix ? take(static_cast<size_t>(c->num_heads) * L.nfix * D * 2) : SIZE_MAX;
  L.vfix = L.nfix ? take(static_cast<size_t>(c->num_heads) * L.nfix * D * 2) : SIZE_MAX;
  L.ofix = L.nfix ? take(qrows * D * 4) : SIZE_MAX;
  L.lsefix = L.nfix ? take(qrows * 4) : SIZE_MAX;
  L.kbits_words = (!d.fp32 && d.pads) ? static_cast<size_t>(attn_tc_tiles(d.img_per_head)) * 4 : 0;
  L.kbits = L.kbits_words ? take(L.kbits_words * 4) : SIZE_MAX;
  const long long n_dense = static_cast<long long>(c->num_frames) * (c->num_special + c->pad_h * c->pad_w);
  L.kbits_dense_words = (!d.fp32 && d.pads && n_dense < (1LL << 31)) ? static_cast<size_t>(attn_tc_tiles(n_dense)) * 4 : 0;
  L.kbits_dense = L.kbits_dense_words ? take(L.kbits_dense_words * 4) : SIZE_MAX;
  L.ngroups = sel_on_tc(c, d) ? sel_group_count(d.R) : 0;
  L.winof = L.ngroups ? take(static_cast<size_t>(d.R) * 4) : SIZE_MAX;
  L.grpof = L.ngroups ? take(static_cast<size_t>(L.ngroups) * 4) : SIZE_MAX;
  L.uni = L.ngroups ? take(static_cast<size_t>(c->num_heads) * L.ngroups * SEL_GROUP * c->topk * 8) : SIZE_MAX;
  L.ucnt = L.ngroups ? take(static_cast<size_t>(c->num_heads) * L.ngroups * 4) : SIZE_MAX;
  L.total = off;
  return L;
}

}  // namespace

struct gsa_ctx {
  gsa_config cfg;
  int fixed[GSA_MAX_FIXED_FRAMES];
  Derived d;
  Layout L;
  int device;
  uint8_t* ws;
  cudaStream_t last_stream;
  int profiling;
  cudaEvent_t ev[MAX_EVENTS];
  const char* ev_names[MAX_EVENTS];
  int n_ev;
  // host-buffer path (gsa_forward_host): device copies of one call's inputs and
  // outputs, copy streams and per-chunk events, created on first use
  uint8_t* stage;
  size_t stage_bytes;
  uint8_t* bw;                 // backward scratch (gsa_backward), created on first use
  size_t bw_bytes;
  cudaStream_t s_in, s_out;
  cudaEvent_t ev_start, ev_in[MAX_CHUNKS], ev_comp[MAX_CHUNKS], ev_out;
  template <typename T>
  T* at(size_t off) const { return off == SIZE_MAX ? nullptr : reinterpret_cast<T*>(ws + off); }
};

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// the variants fix the blend: no compressed value -> O_sel, no selection ->
// O_comp; the descriptor attention has no gate at all
int effective_gate(const gsa_config& c) {
  if (c.variant == GSA_VARIANT_NO_COMP_VALUE) return GSA_GATE_SEL_ONLY;
  if (c.variant == GSA_VARIANT_NO_SELECTION || c.variant == GSA_VARIANT_DESCRIPTOR) return GSA_GATE_COMP_ONLY;
  return c.gate_mode;
}

float scale_of(const gsa_config& c) {
  return c.softmax_scale > 0.f ? c.softmax_scale : 1.f / sqrtf(static_cast<float>(c.head_dim));
}

Grid grid_of(const gsa_config& c) {
  Grid g;
  g.Hp = c.pad_h; g.Wp = c.pad_w; g.Hv = c.grid_h; g.Wv = c.grid_w; g.ns = c.num_special;
  return g;
}

// records an event after a kernel when profiling is on
struct Prof {
  gsa_ctx* ctx;
  cudaStream_t st;
  bool on;
  Prof(gsa_ctx* c, cudaStream_t s, bool timing = true)
      : ctx(c), st(s), on(timing && (c->profiling & GSA_PROFILE_TIMES)) {
    if (!on) return;
    ctx->n_ev = 0;
    cudaEventRecord(ctx->ev[ctx->n_ev++], st);
  }
  void mark(const char* name) {
    if (on && ctx->n_ev < MAX_EVENTS) {
      ctx->ev_names[ctx->n_ev - 1] = name;
      cudaEventRecord(ctx->ev[ctx->n_ev++], st);
    }
  }
};

}  // namespace

extern "C" {

const char* gsa_strerror(int code) {
  switch (code) {
    case GSA_OK: return "ok";
    case GSA_ERR_INVALID_ARG: return "invalid argument";
    case GSA_ERR_SHAPE: return "unsupported or inconsistent shape";
    case GSA_ERR_UNSUPPORTED: return "configuration not supported";
    case GSA_ERR_OOM: return "device workspace allocation failed";
    case GSA_ERR_CUDA: return "CUDA runtime error";
    case GSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case GSA_ERR_DEVICE_BOUNDS: return "device-side index out of bounds";
    default: return "unknown status";
  }
}

size_t gsa_workspace_bytes(const gsa_config* cfg) {
  Derived d;
  if (validate(cfg, &d) != GSA_OK) return 0;
  return make_layout(cfg, d).total;
}

int gsa_create(const gsa_config* cfg, gsa_ctx** out) {
  if (!out) return GSA_ERR_INVALID_ARG;
  *out = nullptr;
  Derived d;
  int rc = validate(cfg, &d);
  if (rc != GSA_OK) return rc;
  gsa_ctx* c = new (std::nothrow) gsa_ctx();
  if (!c) return GSA_ERR_OOM;
  c->cfg = *cfg;
  for (int i = 0; i < cfg->num_fixed_frames; ++i) c->fixed[i] = cfg->fixed_frames[i];
  c->cfg.fixed_frames = c->fixed;
  c->d = d;
  c->L = make_layout(cfg, d);
  if (cudaGetDevice(&c->device) != cudaSuccess) { delete c; return GSA_ERR_CUDA; }
  if (cudaMalloc(&c->ws, c->L.total) != cudaSuccess) {
    cudaGetLastError();
    delete c;
    return GSA_ERR_OOM;
  }
  if (cudaMemset(c->ws + c->L.err, 0, 16) != cudaSuccess) { cudaFree(c->ws); delete c; return GSA_ERR_CUDA; }
  for (int layout = 0; layout < 2; ++layout) {
    // token validity of a padded grid, the same for every head: the image tokens
    // alone (layout 0) or the dense layout, each frame's special tokens first (1)
    const size_t words = layout ? c->L.kbits_dense_words : c->L.kbits_words;
    if (!words) continue;
    const int lead = layout ? cfg->num_special : 0;
    const long long per = lead + static_cast<long long>(cfg->pad_h) * cfg->pad_w;
    const long long n = static_cast<long long>(cfg->num_frames) * per;
    std::vector<uint32_t> bits(words, 0u);
    for (long long t = 0; t < n; ++t) {
      const int o = static_cast<int>(t % per) - lead;
      const bool ok = o < 0 || (o / cfg->pad_w < cfg->grid_h && o % cfg->pad_w < cfg->grid_w);
      if (ok) bits[t >> 5] |= 1u << (t & 31);
    }
    if (cudaMemcpy(c->ws + (layout ? c->L.kbits_dense : c->L.kbits), bits.data(), words * 4,
                   cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(c->ws);
      delete c;
      return GSA_ERR_CUDA;
    }
  }
  if (c->L.ngroups) {
    std::vector<int> order(static_cast<size_t>(d.R));
    sel_group_order(cfg->num_frames, cfg->pad_h / cfg->pool_s, cfg->pad_w / cfg->pool_s, order.data());
    std::vector<int> sched(static_cast<size_t>(c->L.ngroups));
    sel_group_schedule(cfg->num_frames, d.rpf, c->L.ngroups, sched.data());
    if (cudaMemcpy(c->ws + c->L.winof, order.data(), order.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->ws + c->L.grpof, sched.data(), sched.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(c->ws);
      delete c;
      return GSA_ERR_CUDA;
    }
  }
  for (int i = 0; i < MAX_EVENTS; ++i) {
    if (cudaEventCreate(&c->ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(c->ev[j]);
      cudaFree(c->ws);
      delete c;
      return GSA_ERR_CUDA;
    }
  }
  c->last_stream = nullptr;
  *out = c;
  return GSA_OK;
}

void gsa_destroy(gsa_ctx* c) {
  if (!c) return;
  DeviceGuard dg(c->device);
  if (c->bw) cudaFree(c->bw);
  if (c->stage) {
    cudaFree(c->stage);
    cudaStreamDestroy(c->s_in);
    cudaStreamDestroy(c->s_out);
    cudaEventDestroy(c->ev_start);
    cudaEventDestroy(c->ev_out);
    for (int i = 0; i < MAX_CHUNKS; ++i) {
      cudaEventDestroy(c->ev_in[i]);
      cudaEventDestroy(c->ev_comp[i]);
    }
  }
  for (int i = 0; i < MAX_EVENTS; ++i) cudaEventDestroy(c->ev[i]);
  cudaFree(c->ws);
  delete c;
}

}  // extern "C"

namespace {

// The layer for heads [h0, h0 + nh) of the context: every tensor argument
// points at head 0 of its full [H]... array; workspace rows of those heads are
// used, the special-token partials from their start (capacity n_split * H rows
// per query, split count chosen for nh heads within it).
int forward_heads(gsa_ctx* c, int h0, int nh, const void* q_spec, const void* k_spec, const void* v_spec,
                  const void* q_img, const void* k_img, const void* v_img, const void* w_g,
                  void* o_spec, void* o_img, int32_t* sel_idx_out, cudaStream_t st, bool timing) {
  const gsa_config& cf = c->cfg;
  const Derived& d = c->d;
  // the ablation variants fix the blend: no compressed value -> O_sel, no selection -> O_comp
  const int gate = effective_gate(cf);
  const bool no_sel = cf.variant == GSA_VARIANT_NO_SELECTION || cf.variant == GSA_VARIANT_DESCRIPTOR;
  if (gate == GSA_GATE_LEARNED && !w_g) return GSA_ERR_INVALID_ARG;
  if (no_sel && sel_idx_out) return GSA_ERR_INVALID_ARG;
  const int H = nh;
  // per-head strides in bytes, and the views of heads [h0, h0 + nh)
  const size_t es = d.esize;
  const size_t img_b = static_cast<size_t>(d.img_per_head) * D * es;
  const size_t spec_b = static_cast<size_t>(d.spec_per_head) * D * es;
  const size_t rrow = static_cast<size_t>(d.R) * D;
  auto off = [&](const void* p, size_t per_head) -> const void* {
    return p ? static_cast<const uint8_t*>(p) + static_cast<size_t>(h0) * per_head : nullptr;
  };
  auto offm = [&](void* p, size_t per_head) -> void* {
    return p ? static_cast<uint8_t*>(p) + static_cast<size_t>(h0) * per_head : nullptr;
  };
  auto ws = [&](size_t o, size_t per_head) -> uint8_t* {
    return o == SIZE_MAX ? nullptr : c->ws + o + static_cast<size_t>(h0) * per_head;
  };
  q_img = off(q_img, img_b); k_img = off(k_img, img_b); v_img = off(v_img, img_b);
  q_spec = off(q_spec, spec_b); k_spec = off(k_spec, spec_b); v_spec = off(v_spec, spec_b);
  w_g = off(w_g, static_cast<size_t>(D) * D * es);
  o_img = offm(o_img, img_b); o_spec = offm(o_spec, spec_b);
  if (sel_idx_out) sel_idx_out += static_cast<size_t>(h0) * d.R * cf.topk;
  __nv_bfloat16* comp16[3];
  __nv_bfloat16* complo[2];
  float* comp32[3];
  for (int i = 0; i < 3; ++i) {
    comp16[i] = reinterpret_cast<__nv_bfloat16*>(ws(c->L.comp16[i], rrow * 2));
    comp32[i] = reinterpret_cast<float*>(ws(c->L.comp32[i], rrow * 4));
  }
  for (int i = 0; i < 2; ++i) complo[i] = reinterpret_cast<__nv_bfloat16*>(ws(c->L.complo[i], rrow * 2));
  float* ocomp = reinterpret_cast<float*>(ws(c->L.ocomp, rrow * 4));
  int* idx = reinterpret_cast<int*>(ws(c->L.idx, static_cast<size_t>(d.R) * cf.topk * 4));
  uint8_t* osel = ws(c->L.osel, img_b);
  const Grid g = grid_of(cf);
  const float scale = scale_of(cf);
  int* err = c->at<int>(c->L.err);
  if (!k_spec) k_spec = k_img;   // never dereferenced without special/fixed tokens
  if (!v_spec) v_spec = v_img;
  if (!w_g) w_g = q_img;         // never read when the gate is forced
  Prof prof(c, st, timing);

  if (cf.variant == GSA_VARIANT_DESCRIPTOR) {
    // FlashVGGT descriptor attention: descriptors of K and V into the pooled
    // K/V workspace rows, then image queries and special queries attend to
    // [descriptors of every frame ; special tokens of every frame]
    const int Hd = cf.grid_h / cf.pool_s, Wd = cf.grid_w / cf.pool_s;
    const long long ndesc = static_cast<long long>(cf.num_frames) * Hd * Wd;
    // descriptors packed per head ([H][ndesc][64], ndesc <= R): the tensor-core
    // attention addresses key rows as h * n_k + key
    const long long rhs = ndesc * D;
    DescArgs da;
    da.src[0] = k_img; da.src[1] = v_img;
    da.dst[0] = d.fp32 ? static_cast<void*>(comp32[1]) : static_cast<void*>(comp16[1]);
    da.dst[1] = d.fp32 ? static_cast<void*>(comp32[2]) : static_cast<void*>(comp16[2]);
    da.dst_hs = rhs;
    da.H = H; da.F = cf.num_frames; da.Hp = cf.pad_h; da.Wp = cf.pad_w; da.Hv = cf.grid_h; da.Wv = cf.grid_w;
    da.Hd = Hd; da.Wd = Wd;
    if (launch_descriptors(da, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("descriptors");
    const long long shs = d.spec_per_head * D, ihs = d.img_per_head * D;
    const int spec_tiles = attn_tc_tiles(d.spec_per_head);
    const int dtiles = attn_tc_tiles(ndesc);
    for (int pass = 0; pass < 2; ++pass) {
      // pass 0: image queries (one key split: plenty of CTAs); pass 1: special queries
      if (pass == 1 && cf.num_special == 0) break;
      const long long nq = pass == 0 ? d.img_per_head : d.spec_per_head;
      const long long qhs = pass == 0 ? ihs : shs;
      const void* qp = pass == 0 ? q_img : q_spec;
      void* op = pass == 0 ? o_img : o_spec;
      const int qmask = (pass == 0 && d.pads) ? MASK_IMG : MASK_NONE;
      const int nseg = cf.num_special > 0 ? 2 : 1;
      const int ttot = dtiles + (nseg > 1 ? spec_tiles : 0);
      int tps = ttot, nsplit = 1;
      if (pass == 1) {
        attn_tc_split(H, nq, ttot, &tps, &nsplit);
        const int cap = static_cast<int>((static_cast<long long>(d.spec_split) * cf.num_heads) / H);
        if (nsplit > cap) {
          tps = (ttot + cap - 1) / cap;
          nsplit = (ttot + tps - 1) / tps;
        }
      }
      if (!d.fp32) {
        AttnArgs a;
        memset(&a, 0, sizeof(a));
        a.q = reinterpret_cast<const __nv_bfloat16*>(qp); a.q_hs = qhs; a.n_q = static_cast<int>(nq);
        a.q_mask = qmask;
        a.nseg = nseg;
        a.k[0] = comp16[1]; a.v[0] = comp16[2]; a.kv_hs[0] = rhs; a.n_k[0] = static_cast<int>(ndesc);
        a.kmask[0] = MASK_NONE;
        a.k[1] = reinterpret_cast<const __nv_bfloat16*>(k_spec);
        a.v[1] = reinterpret_cast<const __nv_bfloat16*>(v_spec);
        a.kv_hs[1] = shs; a.n_k[1] = static_cast<int>(d.spec_per_head); a.kmask[1] = MASK_NONE;
        a.tiles0 = dtiles; a.tiles_total = ttot; a.tiles_per_split = tps; a.n_split = nsplit;
        a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
        a.o16 = reinterpret_cast<__nv_bfloat16*>(op); a.o_hs = qhs;
        a.part_o = c->at<float>(c->L.part_o); a.part_ml = c->at<float>(c->L.part_ml);
        a.err = err;
        if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
        if (nsplit > 1) {
          MergeArgs m;
          m.lse = nullptr;
          m.part_o = a.part_o; m.part_ml = a.part_ml; m.n_split = nsplit; m.H = H;
          m.n_q = a.n_q; m.scale_log2 = a.scale_log2; m.o16 = a.o16; m.o32 = nullptr; m.o_hs = qhs;
          if (launch_merge(m, st) != cudaSuccess) return GSA_ERR_CUDA;
        }
      } else {
        AttnF32Args a;
        memset(&a, 0, sizeof(a));
        a.q = reinterpret_cast<const float*>(qp); a.q_hs = qhs; a.n_q = static_cast<int>(nq); a.q_mask = qmask;
        a.nseg = nseg;
        a.k[0] = comp32[1]; a.v[0] = comp32[2]; a.kv_hs[0] = rhs; a.n_k[0] = static_cast<int>(ndesc);
        a.kmask[0] = MASK_NONE;
        a.k[1] = reinterpret_cast<const float*>(k_spec); a.v[1] = reinterpret_cast<const float*>(v_spec);
        a.kv_hs[1] = shs; a.n_k[1] = static_cast<int>(d.spec_per_head); a.kmask[1] = MASK_NONE;
        a.H = H; a.g = g; a.scale = scale;
        a.o = reinterpret_cast<float*>(op); a.o_hs = qhs;
        if (launch_attn_f32(a, false, st) != cudaSuccess) return GSA_ERR_CUDA;
      }
      prof.mark(pass == 0 ? "descriptor_attn_img" : "descriptor_attn_spec");
    }
    return GSA_OK;
  }

  // K1 pool
  PoolArgs pa;
  pa.src[0] = q_img; pa.src[1] = k_img; pa.src[2] = v_img;
  for (int i = 0; i < 3; ++i) {
    pa.out16[i] = comp16[i];
    pa.outlo[i] = i < 2 ? complo[i] : nullptr;
    pa.out32[i] = comp32[i];
  }
  pa.H = H; pa.F = cf.num_frames; pa.Hp = cf.pad_h; pa.Wp = cf.pad_w;
  pa.Hv = cf.grid_h; pa.Wv = cf.grid_w; pa.s = cf.pool_s;
  if (launch_pool(pa, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
  prof.mark("pool");

  // K2 compressed attention + streaming top-k
  const long long rhs = static_cast<long long>(d.R) * D;
  if (!d.fp32) {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.q = comp16[0]; a.q_hs = rhs; a.n_q = d.R; a.q_mask = MASK_NONE;
    a.q_lo = complo[0]; a.k_lo = complo[1];
    a.nseg = 1;
    a.k[0] = a.k[1] = comp16[1];
    a.v[0] = a.v[1] = comp16[2];
    a.kv_hs[0] = a.kv_hs[1] = rhs; a.n_k[0] = a.n_k[1] = d.R;
    a.kmask[0] = a.kmask[1] = MASK_NONE;
    a.tiles0 = a.tiles_total = a.tiles_per_split = attn_tc_tiles(d.R); a.n_split = 1;
    a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
    a.o32 = ocomp; a.o_hs = rhs;
    // the top-k runs in passes of at most 32 regions per row: the first pass is fused
    // with the attention, each later pass is a guide-only launch that continues the
    // sorted selection after the previous pass's last entry of the row
    const int kt = no_sel ? 0 : d.kc;
    a.kc = kt < 32 ? kt : 32; a.cand = idx; a.cand_user = sel_idx_out;
    a.cand_stride = kt; a.cand_off = 0;
    float* last_s = reinterpret_cast<float*>(ws(c->L.last_s, static_cast<size_t>(d.R) * 4));
    int* last_i = reinterpret_cast<int*>(ws(c->L.last_i, static_cast<size_t>(d.R) * 4));
    if (kt > 32) { a.last_s = last_s; a.last_i = last_i; }
    a.guide_only = cf.variant == GSA_VARIANT_NO_COMP_VALUE ? 1 : 0;
    a.lse = reinterpret_cast<float*>(ws(c->L.lse_c, static_cast<size_t>(d.R) * 4));
    a.rpf = d.rpf; a.n_fixed = cf.num_fixed_frames;
    for (int i = 0; i < cf.num_fixed_frames; ++i) a.fixed[i] = c->fixed[i];
    a.err = err;
    if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
    for (int off0 = 32; off0 < kt; off0 += 32) {
      AttnArgs b = a;
      b.guide_only = 1;
      b.kc = kt - off0 < 32 ? kt - off0 : 32;
      b.cand_off = off0;
      b.excl_s = last_s; b.excl_i = last_i;          // read and rewritten row by row
      b.last_s = off0 + 32 < kt ? last_s : nullptr;
      b.last_i = off0 + 32 < kt ? last_i : nullptr;
      b.o32 = nullptr; b.lse = nullptr;
      if (launch_attn_tc(b, st) != cudaSuccess) return GSA_ERR_CUDA;
    }
  } else {
    AttnF32Args a;
    memset(&a, 0, sizeof(a));
    a.q = comp32[0]; a.q_hs = rhs; a.n_q = d.R; a.q_mask = MASK_NONE;
    a.nseg = 1;
    a.k[0] = a.k[1] = comp32[1];
    a.v[0] = a.v[1] = comp32[2];
    a.kv_hs[0] = a.kv_hs[1] = rhs; a.n_k[0] = a.n_k[1] = d.R;
    a.H = H; a.g = g; a.scale = scale;
    a.o = ocomp; a.o_hs = rhs;
    a.kc = d.kc; a.cand = idx; a.cand_user = sel_idx_out;
    a.rpf = d.rpf; a.n_fixed = cf.num_fixed_frames;
    for (int i = 0; i < cf.num_fixed_frames; ++i) a.fixed[i] = c->fixed[i];
    if (launch_attn_f32(a, !no_sel, st) != cudaSuccess) return GSA_ERR_CUDA;
  }
  prof.mark(no_sel ? "comp_attn" : cf.variant == GSA_VARIANT_NO_COMP_VALUE ? "comp_guide_topk" : "comp_attn_topk");

  // K3 selection (+ K4 upsample/gate/blend, fused for bf16)
  SelArgs sa;
  sa.q_img = q_img; sa.k_img = k_img; sa.v_img = v_img; sa.k_spec = k_spec; sa.v_spec = v_spec;
  sa.idx = idx; sa.o_sel = osel;
  sa.H = H; sa.F = cf.num_frames; sa.R = d.R; sa.rpf = d.rpf; sa.topk = cf.topk; sa.s = cf.pool_s;
  sa.g = g; sa.scale_log2 = scale * LOG2E; sa.n_fixed = cf.num_fixed_frames;
  for (int i = 0; i < cf.num_fixed_frames; ++i) sa.fixed[i] = c->fixed[i];
  sa.fix_o = nullptr; sa.fix_lse = nullptr;
  sa.err = err;
  EpiArgs ea;
  ea.q_img = q_img; ea.o_sel = osel; ea.o_comp = ocomp;
  ea.w_g = w_g; ea.o_img = o_img; ea.H = H; ea.F = cf.num_frames; ea.R = d.R; ea.rpf = d.rpf;
  ea.s = cf.pool_s; ea.g = g; ea.gate_mode = gate;
  if (no_sel) {
    // no selection branch: the epilogue only upsamples O'_comp (O_sel is never read)
    ea.o_sel = nullptr;
    if (launch_epilogue(ea, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("upsample");
  } else if (!d.fp32) {
    // O_sel is written only when the caller asked to keep intermediates
    if (!(c->profiling & GSA_PROFILE_KEEP_OSEL)) sa.o_sel = nullptr;
    if (c->L.nfix > 0) {
      // the fixed frames' tokens are keys of every window: one dense tensor-core
      // attention of all image queries over them, merged into each window's
      // softmax over its selected regions by the two log-sum-exps
      const long long nfix = c->L.nfix;
      const size_t qrows = static_cast<size_t>(d.img_per_head);
      auto* kfix = reinterpret_cast<__nv_bfloat16*>(ws(c->L.kfix, static_cast<size_t>(nfix) * D * 2));
      auto* vfix = reinterpret_cast<__nv_bfloat16*>(ws(c->L.vfix, static_cast<size_t>(nfix) * D * 2));
      float* ofix = reinterpret_cast<float*>(ws(c->L.ofix, qrows * D * 4));
      float* lsefix = reinterpret_cast<float*>(ws(c->L.lsefix, qrows * 4));
      if (launch_fixed_gather(sa, kfix, vfix, st) != cudaSuccess) return GSA_ERR_CUDA;
      AttnArgs a;
      memset(&a, 0, sizeof(a));
      a.q = reinterpret_cast<const __nv_bfloat16*>(q_img); a.q_hs = static_cast<long long>(qrows) * D;
      a.n_q = static_cast<int>(qrows); a.q_mask = MASK_NONE;
      a.nseg = 1;
      a.k[0] = a.k[1] = kfix; a.v[0] = a.v[1] = vfix;
      a.kv_hs[0] = a.kv_hs[1] = nfix * D; a.n_k[0] = a.n_k[1] = static_cast<int>(nfix);
      a.kmask[0] = a.kmask[1] = MASK_NONE;
      a.tiles0 = a.tiles_total = a.tiles_per_split = attn_tc_tiles(nfix); a.n_split = 1;
      a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
      a.o32 = ofix; a.o_hs = static_cast<long long>(qrows) * D;
      a.lse = lsefix;
      a.err = err;
      if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
      prof.mark("fixed_attn");
      sa.fix_o = ofix; sa.fix_lse = lsefix;
    }
    if (c->L.ngroups) {
      // groups of 8 neighbouring windows on the tensor cores: the union of their
      // regions, then one CTA per group
      SelTcArgs ta;
      memset(&ta, 0, sizeof(ta));
      ta.q_img = q_img; ta.k_img = k_img; ta.v_img = v_img; ta.w_g = w_g;
      ta.idx = idx;
      ta.win_of = c->at<const int>(c->L.winof);
      ta.grp_of = c->at<const int>(c->L.grpof);
      ta.NG = c->L.ngroups;
      ta.topk = cf.topk;
      ta.emax = SEL_GROUP * cf.topk;
      ta.uni = reinterpret_cast<uint2*>(ws(c->L.uni, static_cast<size_t>(ta.NG) * ta.emax * 8));
      ta.ucnt = reinterpret_cast<int*>(ws(c->L.ucnt, static_cast<size_t>(ta.NG) * 4));
      ta.o_comp = ocomp; ta.fix_o = sa.fix_o; ta.fix_lse = sa.fix_lse;
      ta.o_img = static_cast<__nv_bfloat16*>(o_img);
      ta.o_sel = static_cast<__nv_bfloat16*>(sa.o_sel);
      ta.H = H; ta.F = cf.num_frames; ta.R = d.R; ta.rpf = d.rpf; ta.rx = cf.pad_w / cf.pool_s;
      ta.g = g; ta.scale_log2 = scale * LOG2E; ta.gate_mode = gate;
      ta.err = err;
      if (launch_sel_union(ta, st) != cudaSuccess) return GSA_ERR_CUDA;
      prof.mark("sel_union");
      if (launch_sel_tc(ta, st) != cudaSuccess) return GSA_ERR_CUDA;
    } else if (launch_sel_fused(sa, ea, st) != cudaSuccess) {
      return GSA_ERR_CUDA;
    }
    prof.mark("selection_gate");
  } else {
    if (launch_sel(sa, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("selection");
    if (launch_epilogue(ea, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("epilogue");
  }

  // K5 special tokens over every token; the split count fills the GPU for nh
  // heads, within the partials' capacity (d.spec_split splits of all H heads)
  int tps = d.spec_tps, nsplit = d.spec_split;
  if (nh != cf.num_heads && cf.num_special > 0) {
    attn_tc_split(nh, d.spec_per_head, d.spec_tiles_total, &tps, &nsplit);
    const int cap = static_cast<int>((static_cast<long long>(d.spec_split) * cf.num_heads) / nh);
    if (nsplit > cap) {
      tps = (d.spec_tiles_total + cap - 1) / cap;
      nsplit = (d.spec_tiles_total + tps - 1) / tps;
    }
  }
  if (cf.num_special > 0) {
    const long long shs = d.spec_per_head * D;
    const long long ihs = d.img_per_head * D;
    if (!d.fp32) {
      AttnArgs a;
      memset(&a, 0, sizeof(a));
      a.q = reinterpret_cast<const __nv_bfloat16*>(q_spec); a.q_hs = shs;
      a.n_q = static_cast<int>(d.spec_per_head); a.q_mask = MASK_NONE;
      a.nseg = 2;
      a.k[0] = reinterpret_cast<const __nv_bfloat16*>(k_spec);
      a.v[0] = reinterpret_cast<const __nv_bfloat16*>(v_spec);
      a.kv_hs[0] = shs; a.n_k[0] = static_cast<int>(d.spec_per_head); a.kmask[0] = MASK_NONE;
      a.k[1] = reinterpret_cast<const __nv_bfloat16*>(k_img);
      a.v[1] = reinterpret_cast<const __nv_bfloat16*>(v_img);
      a.kv_hs[1] = ihs; a.n_k[1] = static_cast<int>(d.img_per_head);
      a.kmask[1] = d.pads ? MASK_IMG : MASK_NONE;
      a.kbits[1] = c->at<const uint32_t>(c->L.kbits);
      a.tiles0 = d.spec_tiles0; a.tiles_total = d.spec_tiles_total;
      a.tiles_per_split = tps; a.n_split = nsplit;
      a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
      a.o16 = reinterpret_cast<__nv_bfloat16*>(o_spec); a.o_hs = shs;
      a.part_o = c->at<float>(c->L.part_o); a.part_ml = c->at<float>(c->L.part_ml);
      a.lse = reinterpret_cast<float*>(ws(c->L.lse_s, static_cast<size_t>(d.spec_per_head) * 4));
      a.err = err;
      if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
      prof.mark("special");
      if (nsplit > 1) {
        MergeArgs m;
        m.lse = nullptr;
        m.part_o = a.part_o; m.part_ml = a.part_ml; m.n_split = nsplit; m.H = H;
        m.n_q = a.n_q; m.scale_log2 = a.scale_log2; m.o16 = a.o16; m.o32 = nullptr; m.o_hs = shs;
        m.lse = a.lse;
        if (launch_merge(m, st) != cudaSuccess) return GSA_ERR_CUDA;
        prof.mark("special_merge");
      }
    } else {
      AttnF32Args a;
      memset(&a, 0, sizeof(a));
      a.q = reinterpret_cast<const float*>(q_spec); a.q_hs = shs;
      a.n_q = static_cast<int>(d.spec_per_head); a.q_mask = MASK_NONE;
      a.nseg = 2;
      a.k[0] = reinterpret_cast<const float*>(k_spec); a.v[0] = reinterpret_cast<const float*>(v_spec);
      a.kv_hs[0] = shs; a.n_k[0] = static_cast<int>(d.spec_per_head); a.kmask[0] = MASK_NONE;
      a.k[1] = reinterpret_cast<const float*>(k_img); a.v[1] = reinterpret_cast<const float*>(v_img);
      a.kv_hs[1] = ihs; a.n_k[1] = static_cast<int>(d.img_per_head);
      a.kmask[1] = d.pads ? MASK_IMG : MASK_NONE;
      a.H = H; a.g = g; a.scale = scale;
      a.o = reinterpret_cast<float*>(o_spec); a.o_hs = shs;
      if (launch_attn_f32(a, false, st) != cudaSuccess) return GSA_ERR_CUDA;
      prof.mark("special");
    }
  }
  return GSA_OK;
}

}  // namespace

extern "C" {

int gsa_forward(gsa_ctx* c, const void* q_spec, const void* k_spec, const void* v_spec,
                const void* q_img, const void* k_img, const void* v_img, const void* w_g,
                void* o_spec, void* o_img, int32_t* sel_idx_out, void* stream) {
  if (!c || !q_img || !k_img || !v_img || !o_img) return GSA_ERR_INVALID_ARG;
  const gsa_config& cf = c->cfg;
  if (cf.num_special > 0 && (!q_spec || !k_spec || !v_spec || !o_spec)) return GSA_ERR_INVALID_ARG;
  const int gate = effective_gate(cf);
  if (gate == GSA_GATE_LEARNED && !w_g) return GSA_ERR_INVALID_ARG;
  if (cf.variant == GSA_VARIANT_NO_SELECTION && sel_idx_out) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  c->last_stream = st;
  return forward_heads(c, 0, cf.num_heads, q_spec, k_spec, v_spec, q_img, k_img, v_img, w_g, o_spec, o_img,
                       sel_idx_out, st, true);
}

int gsa_forward_host(gsa_ctx* c, const void* q_spec, const void* k_spec, const void* v_spec,
                     const void* q_img, const void* k_img, const void* v_img, const void* w_g,
                     void* o_spec, void* o_img, int32_t* sel_idx_out, void* stream) {
  if (!c || !q_img || !k_img || !v_img || !o_img) return GSA_ERR_INVALID_ARG;
  const gsa_config& cf = c->cfg;
  const Derived& d = c->d;
  const bool spec = cf.num_special > 0;
  if (spec && (!q_spec || !k_spec || !v_spec || !o_spec)) return GSA_ERR_INVALID_ARG;
  const int gate = effective_gate(cf);
  if (gate == GSA_GATE_LEARNED && !w_g) return GSA_ERR_INVALID_ARG;
  if (cf.variant == GSA_VARIANT_NO_SELECTION && sel_idx_out) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int H = cf.num_heads;
  const size_t es = d.esize;
  const size_t img_b = static_cast<size_t>(d.img_per_head) * D * es;
  const size_t spec_b = static_cast<size_t>(d.spec_per_head) * D * es;
  const size_t wg_b = static_cast<size_t>(D) * D * es;
  const size_t idx_b = static_cast<size_t>(d.R) * cf.topk * 4;
  const bool wg = gate == GSA_GATE_LEARNED;
  // device copies: q/k/v_img, q/k/v_spec, w_g, o_img, o_spec, idx ([H]... each)
  size_t offs[10], tot = 0;
  const size_t per[10] = {img_b, img_b, img_b, spec_b, spec_b, spec_b, wg_b, img_b, spec_b, idx_b};
  for (int i = 0; i < 10; ++i) {
    offs[i] = tot;
    tot = align_up(tot + per[i] * H);
  }
  if (!c->stage) {
    if (cudaMalloc(&c->stage, tot) != cudaSuccess) {
      c->stage = nullptr;
      return GSA_ERR_OOM;
    }
    c->stage_bytes = tot;
    if (cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c->s_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_out, cudaEventDisableTiming) != cudaSuccess)
      return GSA_ERR_CUDA;
    for (int i = 0; i < MAX_CHUNKS; ++i)
      if (cudaEventCreateWithFlags(&c->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&c->ev_comp[i], cudaEventDisableTiming) != cudaSuccess)
        return GSA_ERR_CUDA;
  }
  uint8_t* dp[10];
  for (int i = 0; i < 10; ++i) dp[i] = c->stage + offs[i];
  const void* hin[7] = {q_img, k_img, v_img, q_spec, k_spec, v_spec, w_g};
  // chunks of heads: copies of chunk i+1 in overlap the layer on chunk i, whose
  // outputs go back while chunk i+1 computes
  const int nchunk = H < MAX_CHUNKS ? H : MAX_CHUNKS;
  const int hpc = (H + nchunk - 1) / nchunk;
  if (cudaEventRecord(c->ev_start, st) != cudaSuccess) return GSA_ERR_CUDA;
  if (cudaStreamWaitEvent(c->s_in, c->ev_start, 0) != cudaSuccess) return GSA_ERR_CUDA;
  int k = 0;
  for (int h0 = 0; h0 < H; h0 += hpc, ++k) {
    const int nh = (h0 + hpc <= H) ? hpc : H - h0;
    for (int i = 0; i < 7; ++i) {
      if ((i >= 3 && i < 6 && !spec) || (i == 6 && !wg) || per[i] == 0) continue;
      if (cudaMemcpyAsync(dp[i] + h0 * per[i], static_cast<const uint8_t*>(hin[i]) + h0 * per[i], nh * per[i],
                          cudaMemcpyHostToDevice, c->s_in) != cudaSuccess)
        return GSA_ERR_CUDA;
    }
    if (cudaEventRecord(c->ev_in[k], c->s_in) != cudaSuccess) return GSA_ERR_CUDA;
    if (cudaStreamWaitEvent(st, c->ev_in[k], 0) != cudaSuccess) return GSA_ERR_CUDA;
    const int rc = forward_heads(c, h0, nh, spec ? dp[3] : nullptr, spec ? dp[4] : nullptr, spec ? dp[5] : nullptr,
                                 dp[0], dp[1], dp[2], wg ? dp[6] : nullptr, spec ? dp[8] : nullptr, dp[7],
                                 sel_idx_out ? reinterpret_cast<int32_t*>(dp[9]) : nullptr, st, false);
    if (rc != GSA_OK) return rc;
    if (cudaEventRecord(c->ev_comp[k], st) != cudaSuccess) return GSA_ERR_CUDA;
    if (cudaStreamWaitEvent(c->s_out, c->ev_comp[k], 0) != cudaSuccess) return GSA_ERR_CUDA;
    void* hout[3] = {o_img, spec ? o_spec : nullptr, sel_idx_out};
    const int src[3] = {7, 8, 9};
    for (int i = 0; i < 3; ++i) {
      if (!hout[i] || per[src[i]] == 0) continue;
      if (cudaMemcpyAsync(static_cast<uint8_t*>(hout[i]) + h0 * per[src[i]], dp[src[i]] + h0 * per[src[i]],
                          nh * per[src[i]], cudaMemcpyDeviceToHost, c->s_out) != cudaSuccess)
        return GSA_ERR_CUDA;
    }
  }
  // the caller's stream completes when the last output has reached the host
  if (cudaEventRecord(c->ev_out, c->s_out) != cudaSuccess) return GSA_ERR_CUDA;
  if (cudaStreamWaitEvent(st, c->ev_out, 0) != cudaSuccess) return GSA_ERR_CUDA;
  c->last_stream = st;
  return GSA_OK;
}

int gsa_backward(gsa_ctx* c, const void* q_spec, const void* k_spec, const void* v_spec, const void* q_img,
                 const void* k_img, const void* v_img, const void* w_g, const void* o_spec, const void* d_o_spec,
                 const void* d_o_img, float* dq_spec, float* dk_spec, float* dv_spec, float* dq_img, float* dk_img,
                 float* dv_img, float* dw_g, void* stream) {
  if (!c || !q_img || !k_img || !v_img || !d_o_img || !dq_img || !dk_img || !dv_img || !dw_g)
    return GSA_ERR_INVALID_ARG;
  const gsa_config& cf = c->cfg;
  const Derived& d = c->d;
  const bool spec = cf.num_special > 0;
  if (spec && (!q_spec || !k_spec || !v_spec || !o_spec || !d_o_spec || !dq_spec || !dk_spec || !dv_spec))
    return GSA_ERR_INVALID_ARG;
  if (d.fp32 || cf.variant != GSA_VARIANT_FULL || cf.topk > 64) return GSA_ERR_UNSUPPORTED;
  const int gate = effective_gate(cf);
  if (gate == GSA_GATE_LEARNED && !w_g) return GSA_ERR_INVALID_ARG;
  if (cf.num_fixed_frames > 0 && !spec) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  c->last_stream = st;
  const int H = cf.num_heads;
  const size_t rows = static_cast<size_t>(H) * d.R;
  const size_t img = static_cast<size_t>(H) * d.img_per_head;
  const size_t sp = static_cast<size_t>(H) * d.spec_per_head;
  // scratch: dO'_comp fp32 + bf16, D of compressed and special rows, dQ/dK/dV_comp, da;
  // with the fixed context computed apart (bf16 forward with fixed frames) also dO_sel
  // (bf16), the union log-sum-exp and D of every image token, and dK/dV of the packed
  // fixed keys
  const long long nfix = c->L.nfix;
  const size_t fk = static_cast<size_t>(H) * static_cast<size_t>(nfix);
  size_t off[13], tot = 0;
  const size_t sz[13] = {rows * D * 4, rows * D * 2, rows * 4, sp * 4, rows * D * 4, rows * D * 4, rows * D * 4,
                         img * D * 4, nfix ? img * D * 2 : 0, nfix ? img * 4 : 0, nfix ? img * 4 : 0, fk * D * 4,
                         fk * D * 4};
  for (int i = 0; i < 13; ++i) {
    off[i] = tot;
    tot = align_up(tot + sz[i]);
  }
  if (!c->bw) {
    if (cudaMalloc(&c->bw, tot) != cudaSuccess) {
      c->bw = nullptr;
      return GSA_ERR_OOM;
    }
    c->bw_bytes = tot;
  }
  float* docomp = reinterpret_cast<float*>(c->bw + off[0]);
  __nv_bfloat16* docomp16 = reinterpret_cast<__nv_bfloat16*>(c->bw + off[1]);
  float* Dc = reinterpret_cast<float*>(c->bw + off[2]);
  float* Ds = reinterpret_cast<float*>(c->bw + off[3]);
  float* dqc = reinterpret_cast<float*>(c->bw + off[4]);
  float* dkc = reinterpret_cast<float*>(c->bw + off[5]);
  float* dvc = reinterpret_cast<float*>(c->bw + off[6]);
  float* da = reinterpret_cast<float*>(c->bw + off[7]);
  const Grid g = grid_of(cf);
  const float scale = scale_of(cf);
  int* err = c->at<int>(c->L.err);
  if (!k_spec) k_spec = k_img;
  if (!v_spec) v_spec = v_img;
  if (!w_g) w_g = q_img;
  Prof prof(c, st);
  // gradients reached by atomics or accumulation start at zero
  if (cudaMemsetAsync(dk_img, 0, img * D * 4, st) != cudaSuccess || cudaMemsetAsync(dv_img, 0, img * D * 4, st) != cudaSuccess)
    return GSA_ERR_CUDA;
  // 8 x 8 windows span four warps of the selection backward, which add into dO'_comp
  if (cf.pool_s == 8 && cudaMemsetAsync(docomp, 0, rows * D * 4, st) != cudaSuccess) return GSA_ERR_CUDA;
  if (spec && (cudaMemsetAsync(dk_spec, 0, sp * D * 4, st) != cudaSuccess ||
               cudaMemsetAsync(dv_spec, 0, sp * D * 4, st) != cudaSuccess))
    return GSA_ERR_CUDA;

  // 1. selection branch and gate (windows), dO'_comp, dq of the image tokens
  SelBwdArgs sb;
  memset(&sb, 0, sizeof(sb));
  SelArgs& sa = sb.s;
  sa.q_img = q_img; sa.k_img = k_img; sa.v_img = v_img; sa.k_spec = k_spec; sa.v_spec = v_spec;
  sa.idx = c->at<int>(c->L.idx); sa.o_sel = nullptr;
  sa.H = H; sa.F = cf.num_frames; sa.R = d.R; sa.rpf = d.rpf; sa.topk = cf.topk; sa.s = cf.pool_s;
  sa.g = g; sa.scale_log2 = scale * LOG2E; sa.n_fixed = cf.num_fixed_frames;
  for (int i = 0; i < cf.num_fixed_frames; ++i) sa.fixed[i] = c->fixed[i];
  sa.err = err;
  sb.w_g = w_g; sb.o_comp = c->at<float>(c->L.ocomp); sb.d_o = reinterpret_cast<const __nv_bfloat16*>(d_o_img);
  sb.gate_mode = gate; sb.dq = dq_img; sb.dk = dk_img; sb.dv = dv_img;
  sb.dk_spec = spec ? dk_spec : nullptr; sb.dv_spec = spec ? dv_spec : nullptr;
  sb.d_ocomp = docomp; sb.da = da;
  if (nfix) {
    // the forward attended the fixed context apart (its O_fix, LSE and packed K/V are
    // still in the workspace): the selection backward takes the selected regions only
    sa.fix_o = c->at<float>(c->L.ofix);
    sa.fix_lse = c->at<float>(c->L.lsefix);
    sb.dosel = reinterpret_cast<__nv_bfloat16*>(c->bw + off[8]);
    sb.lse_u = reinterpret_cast<float*>(c->bw + off[9]);
    sb.Dq = reinterpret_cast<float*>(c->bw + off[10]);
  }
  if (launch_sel_bwd(sb, st) != cudaSuccess) return GSA_ERR_CUDA;
  prof.mark("bwd_selection_gate");
  if (nfix) {
    // the fixed context: dense attention backward of every image query over the packed
    // fixed keys, P normalised over the union (its LSE from the selection backward);
    // dq adds to the selection's, dK/dV go back to the fixed frames' tokens
    const long long nq = d.img_per_head;
    float* dkfix = reinterpret_cast<float*>(c->bw + off[11]);
    float* dvfix = reinterpret_cast<float*>(c->bw + off[12]);
    BwdArgs bf;
    memset(&bf, 0, sizeof(bf));
    bf.q = reinterpret_cast<const __nv_bfloat16*>(q_img); bf.q_hs = nq * D; bf.n_q = static_cast<int>(nq);
    bf.nseg = 1;
    bf.k[0] = c->at<__nv_bfloat16>(c->L.kfix); bf.v[0] = c->at<__nv_bfloat16>(c->L.vfix);
    bf.kv_hs[0] = nfix * D; bf.n_k[0] = static_cast<int>(nfix); bf.kmask[0] = MASK_NONE;
    bf.dO = sb.dosel; bf.do_hs = nq * D; bf.lse2 = sb.lse_u; bf.Dv = sb.Dq;
    bf.dq = dq_img; bf.dq_hs = nq * D; bf.dq_accum = 1;
    bf.dk[0] = dkfix; bf.dv[0] = dvfix; bf.dkv_hs[0] = nfix * D; bf.dkv_accum = 0;
    bf.H = H; bf.g = g; bf.scale_log2 = scale * LOG2E; bf.scale = scale;
    if (launch_attn_bwd_dq_tc(bf, err, st) != cudaSuccess || launch_attn_bwd_dkv_tc(bf, err, st) != cudaSuccess)
      return GSA_ERR_CUDA;
    if (launch_fixed_scatter_add(sa, dkfix, dvfix, dk_img, dv_img, dk_spec, dv_spec, st) != cudaSuccess)
      return GSA_ERR_CUDA;
    prof.mark("bwd_fixed_attn");
  }

  // 2. compressed attention (split guide scores, as in the forward)
  const long long rhs = static_cast<long long>(d.R) * D;
  if (launch_rowdot(docomp, nullptr, c->at<float>(c->L.ocomp), nullptr, static_cast<long long>(rows), Dc, docomp16,
                    st) != cudaSuccess)
    return GSA_ERR_CUDA;
  BwdArgs ba;
  memset(&ba, 0, sizeof(ba));
  ba.q = c->at<__nv_bfloat16>(c->L.comp16[0]); ba.q_lo = c->at<__nv_bfloat16>(c->L.complo[0]);
  ba.k_lo = c->at<__nv_bfloat16>(c->L.complo[1]); ba.q_hs = rhs; ba.n_q = d.R; ba.nseg = 1;
  ba.k[0] = c->at<__nv_bfloat16>(c->L.comp16[1]); ba.v[0] = c->at<__nv_bfloat16>(c->L.comp16[2]);
  ba.kv_hs[0] = rhs; ba.n_k[0] = d.R; ba.kmask[0] = MASK_NONE;
  ba.dO = docomp16; ba.do_hs = rhs; ba.lse2 = c->at<float>(c->L.lse_c); ba.Dv = Dc;
  ba.dq = dqc; ba.dq_hs = rhs; ba.dq_accum = 0;
  ba.dk[0] = dkc; ba.dv[0] = dvc; ba.dkv_hs[0] = rhs; ba.dkv_accum = 0;
  ba.H = H; ba.g = g; ba.scale_log2 = scale * LOG2E; ba.scale = scale;
  if (launch_attn_bwd_dq_tc(ba, err, st) != cudaSuccess || launch_attn_bwd_dkv_tc(ba, err, st) != cudaSuccess)
    return GSA_ERR_CUDA;
  prof.mark("bwd_comp_attn");

  // 3. pooling: each valid token takes its region's gradient over the region's size
  PoolBwdArgs pb;
  pb.dcomp[0] = dqc; pb.dcomp[1] = dkc; pb.dcomp[2] = dvc;
  pb.dimg[0] = dq_img; pb.dimg[1] = dk_img; pb.dimg[2] = dv_img;
  pb.H = H; pb.F = cf.num_frames; pb.Hp = cf.pad_h; pb.Wp = cf.pad_w; pb.Hv = cf.grid_h; pb.Wv = cf.grid_w;
  pb.s = cf.pool_s;
  if (launch_pool_bwd(pb, st) != cudaSuccess) return GSA_ERR_CUDA;
  prof.mark("bwd_pool");

  // 4. special tokens over every special and valid image token
  if (spec) {
    const long long shs = d.spec_per_head * D, ihs = d.img_per_head * D;
    if (launch_rowdot(nullptr, reinterpret_cast<const __nv_bfloat16*>(d_o_spec), nullptr,
                      reinterpret_cast<const __nv_bfloat16*>(o_spec), static_cast<long long>(sp), Ds, nullptr,
                      st) != cudaSuccess)
      return GSA_ERR_CUDA;
    BwdArgs bs;
    memset(&bs, 0, sizeof(bs));
    bs.q = reinterpret_cast<const __nv_bfloat16*>(q_spec); bs.q_hs = shs; bs.n_q = static_cast<int>(d.spec_per_head);
    bs.nseg = 2;
    bs.k[0] = reinterpret_cast<const __nv_bfloat16*>(k_spec); bs.v[0] = reinterpret_cast<const __nv_bfloat16*>(v_spec);
    bs.kv_hs[0] = shs; bs.n_k[0] = static_cast<int>(d.spec_per_head); bs.kmask[0] = MASK_NONE;
    bs.k[1] = reinterpret_cast<const __nv_bfloat16*>(k_img); bs.v[1] = reinterpret_cast<const __nv_bfloat16*>(v_img);
    bs.kv_hs[1] = ihs; bs.n_k[1] = static_cast<int>(d.img_per_head); bs.kmask[1] = d.pads ? MASK_IMG : MASK_NONE;
    if (d.pads && c->L.kbits_words) bs.kbits[1] = c->at<const uint32_t>(c->L.kbits);   // the forward's table
    bs.dO = reinterpret_cast<const __nv_bfloat16*>(d_o_spec); bs.do_hs = shs;
    bs.lse2 = c->at<float>(c->L.lse_s); bs.Dv = Ds;
    bs.dq = dq_spec; bs.dq_hs = shs; bs.dq_accum = 0;
    bs.dk[0] = dk_spec; bs.dv[0] = dv_spec; bs.dkv_hs[0] = shs;
    bs.dk[1] = dk_img; bs.dv[1] = dv_img; bs.dkv_hs[1] = ihs; bs.dkv_accum = 1;
    bs.H = H; bs.g = g; bs.scale_log2 = scale * LOG2E; bs.scale = scale;
    if (launch_attn_bwd_dq_tc(bs, err, st) != cudaSuccess || launch_attn_bwd_dkv_tc(bs, err, st) != cudaSuccess)
      return GSA_ERR_CUDA;
    prof.mark("bwd_special");
  }

  // 5. the gate matrix
  if (gate == GSA_GATE_LEARNED) {
    if (launch_dwg(da, reinterpret_cast<const __nv_bfloat16*>(q_img), H, d.img_per_head, dw_g, st) != cudaSuccess)
      return GSA_ERR_CUDA;
  } else if (cudaMemsetAsync(dw_g, 0, static_cast<size_t>(H) * D * D * 4, st) != cudaSuccess) {
    return GSA_ERR_CUDA;
  }
  prof.mark("bwd_gate_weight");
  return GSA_OK;
}

int gsa_dense_forward(gsa_ctx* c, const void* q, const void* k, const void* v, void* o,
                      void* stream) {
  if (!c || !q || !k || !v || !o) return GSA_ERR_INVALID_ARG;
  const gsa_config& cf = c->cfg;
  const Derived& d = c->d;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  c->last_stream = st;
  const long long n = static_cast<long long>(cf.num_frames) * (cf.num_special + cf.pad_h * cf.pad_w);
  if (n >= (1LL << 31)) return GSA_ERR_UNSUPPORTED;
  const long long hs = n * D;
  const Grid g = grid_of(cf);
  const int msk = d.pads ? MASK_DENSE : MASK_NONE;
  Prof prof(c, st);
  if (!d.fp32) {
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.q = reinterpret_cast<const __nv_bfloat16*>(q); a.q_hs = hs; a.n_q = static_cast<int>(n);
    a.q_mask = msk; a.nseg = 1;
    a.k[0] = a.k[1] = reinterpret_cast<const __nv_bfloat16*>(k);
    a.v[0] = a.v[1] = reinterpret_cast<const __nv_bfloat16*>(v);
    a.kv_hs[0] = a.kv_hs[1] = hs; a.n_k[0] = a.n_k[1] = static_cast<int>(n);
    a.kmask[0] = a.kmask[1] = msk;
    a.kbits[0] = a.kbits[1] = c->at<const uint32_t>(c->L.kbits_dense);
    a.tiles0 = a.tiles_total = a.tiles_per_split = attn_tc_tiles(n); a.n_split = 1;
    a.H = cf.num_heads; a.g = g; a.scale_log2 = scale_of(cf) * LOG2E;
    a.o16 = reinterpret_cast<__nv_bfloat16*>(o); a.o_hs = hs;
    a.err = c->at<int>(c->L.err);
    if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
  } else {
    AttnF32Args a;
    memset(&a, 0, sizeof(a));
    a.q = reinterpret_cast<const float*>(q); a.q_hs = hs; a.n_q = static_cast<int>(n);
    a.q_mask = msk; a.nseg = 1;
    a.k[0] = a.k[1] = reinterpret_cast<const float*>(k);
    a.v[0] = a.v[1] = reinterpret_cast<const float*>(v);
    a.kv_hs[0] = a.kv_hs[1] = hs; a.n_k[0] = a.n_k[1] = static_cast<int>(n);
    a.kmask[0] = a.kmask[1] = msk;
    a.H = cf.num_heads; a.g = g; a.scale = scale_of(cf);
    a.o = reinterpret_cast<float*>(o); a.o_hs = hs;
    if (launch_attn_f32(a, false, st) != cudaSuccess) return GSA_ERR_CUDA;
  }
  prof.mark("dense");
  return GSA_OK;
}

int gsa_get_intermediate(gsa_ctx* c, int which, void** dev_ptr, size_t* bytes) {
  if (!c || !dev_ptr || !bytes) return GSA_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(c->cfg.num_heads) * c->d.R;
  size_t off = SIZE_MAX, n = 0;
  switch (which) {
    case 0: case 1: case 2:
      if (c->d.fp32) { off = c->L.comp32[which]; n = rows * D * 4; }
      else { off = c->L.comp16[which]; n = rows * D * 2; }
      break;
    case 3: off = c->L.ocomp; n = rows * D * 4; break;
    case 4: off = c->L.idx; n = rows * c->cfg.topk * 4; break;
    case 5: off = c->L.osel; n = static_cast<size_t>(c->cfg.num_heads) * c->d.img_per_head * D * c->d.esize; break;
    case 6: case 7:
      if (c->d.fp32) { off = c->L.comp32[which - 6]; n = rows * D * 4; }
      else { off = c->L.complo[which - 6]; n = rows * D * 2; }
      break;
    default: return GSA_ERR_INVALID_ARG;
  }
  *dev_ptr = c->ws + off;
  *bytes = n;
  return GSA_OK;
}

int gsa_set_profiling(gsa_ctx* c, int enable) {
  if (!c) return GSA_ERR_INVALID_ARG;
  c->profiling = enable;
  c->n_ev = 0;
  return GSA_OK;
}

int gsa_get_kernel_times(gsa_ctx* c, float* ms, const char** names, int cap) {
  if (!c || cap < 0) return -GSA_ERR_INVALID_ARG;
  if (!(c->profiling & GSA_PROFILE_TIMES) || c->n_ev < 2) return 0;
  DeviceGuard dg(c->device);
  if (cudaEventSynchronize(c->ev[c->n_ev - 1]) != cudaSuccess) return -GSA_ERR_CUDA;
  int n = 0;
  for (int i = 0; i + 1 < c->n_ev && n < cap; ++i, ++n) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, c->ev[i], c->ev[i + 1]) != cudaSuccess) return -GSA_ERR_CUDA;
    if (ms) ms[n] = t;
    if (names) names[n] = c->ev_names[i];
  }
  return n;
}

int gsa_debug_expire_wait(gsa_ctx* c, unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return GSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!c) {
    // no context: the status word of the allocation-free calls on the current device
    int* word = nullptr;
    const int rc = noalloc_status_word(&word);
    if (rc != GSA_OK) return rc;
    return launch_expire_wait(word, 1000ull * limit_us, st) == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
  }
  DeviceGuard dg(c->device);
  if (launch_expire_wait(c->at<int>(c->L.err), 1000ull * limit_us, st) != cudaSuccess) return GSA_ERR_CUDA;
  c->last_stream = st;
  return GSA_OK;
}

int gsa_get_status(gsa_ctx* c) {
  if (!c) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  if (cudaStreamSynchronize(c->last_stream) != cudaSuccess) return GSA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, c->ws + c->L.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GSA_ERR_CUDA;
  if (word != 0 && cudaMemset(c->ws + c->L.err, 0, sizeof(int)) != cudaSuccess) return GSA_ERR_CUDA;
  return word;
}

}  // extern "C"
