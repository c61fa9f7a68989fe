// C ABI of the GSA layer: config validation, workspace ownership, kernel
// sequencing on the caller's stream.  See include/gsa.h for the contract.
#include <math.h>
#include <new>
#include <string.h>

#include "../../include/gsa.h"
#include "gsa_kernels.h"

using namespace gsa;

namespace {

constexpr size_t ALIGN = 256;
constexpr int MAX_EVENTS = 16;

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
  if (c->variant < GSA_VARIANT_FULL || c->variant > GSA_VARIANT_NO_SELECTION) return GSA_ERR_INVALID_ARG;
  if (!(c->softmax_scale >= 0.f) || isinf(c->softmax_scale)) return GSA_ERR_INVALID_ARG;
  if (c->head_dim != 64) return GSA_ERR_SHAPE;
  const int s = c->pool_s;
  if (s != 1 && s != 2 && s != 4 && s != 8) return GSA_ERR_UNSUPPORTED;
  if (c->dtype == GSA_BF16 && s == 8) return GSA_ERR_UNSUPPORTED;
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
  size_t comp16[3], complo[2], comp32[3], ocomp, idx, osel, part_o, part_ml, err, total;
};

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
  L.err = take(16);
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
  Prof(gsa_ctx* c, cudaStream_t s) : ctx(c), st(s) {
    ctx->n_ev = 0;
    if (ctx->profiling & GSA_PROFILE_TIMES) cudaEventRecord(ctx->ev[ctx->n_ev++], st);
  }
  void mark(const char* name) {
    if ((ctx->profiling & GSA_PROFILE_TIMES) && ctx->n_ev < MAX_EVENTS) {
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
  for (int i = 0; i < MAX_EVENTS; ++i) cudaEventDestroy(c->ev[i]);
  cudaFree(c->ws);
  delete c;
}

int gsa_forward(gsa_ctx* c, const void* q_spec, const void* k_spec, const void* v_spec,
                const void* q_img, const void* k_img, const void* v_img, const void* w_g,
                void* o_spec, void* o_img, int32_t* sel_idx_out, void* stream) {
  if (!c || !q_img || !k_img || !v_img || !o_img) return GSA_ERR_INVALID_ARG;
  const gsa_config& cf = c->cfg;
  const Derived& d = c->d;
  if (cf.num_special > 0 && (!q_spec || !k_spec || !v_spec || !o_spec)) return GSA_ERR_INVALID_ARG;
  // the ablation variants fix the blend: no compressed value -> O_sel, no selection -> O_comp
  const int gate = cf.variant == GSA_VARIANT_NO_COMP_VALUE ? GSA_GATE_SEL_ONLY
                   : cf.variant == GSA_VARIANT_NO_SELECTION ? GSA_GATE_COMP_ONLY
                                                            : cf.gate_mode;
  const bool no_sel = cf.variant == GSA_VARIANT_NO_SELECTION;
  if (gate == GSA_GATE_LEARNED && !w_g) return GSA_ERR_INVALID_ARG;
  if (no_sel && sel_idx_out) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  c->last_stream = st;
  const int H = cf.num_heads;
  const Grid g = grid_of(cf);
  const float scale = scale_of(cf);
  int* err = c->at<int>(c->L.err);
  if (!k_spec) k_spec = k_img;   // never dereferenced without special/fixed tokens
  if (!v_spec) v_spec = v_img;
  if (!w_g) w_g = q_img;         // never read when the gate is forced
  Prof prof(c, st);

  // K1 pool
  PoolArgs pa;
  pa.src[0] = q_img; pa.src[1] = k_img; pa.src[2] = v_img;
  for (int i = 0; i < 3; ++i) {
    pa.out16[i] = c->at<__nv_bfloat16>(c->L.comp16[i]);
    pa.outlo[i] = i < 2 ? c->at<__nv_bfloat16>(c->L.complo[i]) : nullptr;
    pa.out32[i] = c->at<float>(c->L.comp32[i]);
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
    a.q = c->at<__nv_bfloat16>(c->L.comp16[0]); a.q_hs = rhs; a.n_q = d.R; a.q_mask = MASK_NONE;
    a.q_lo = c->at<__nv_bfloat16>(c->L.complo[0]); a.k_lo = c->at<__nv_bfloat16>(c->L.complo[1]);
    a.nseg = 1;
    a.k[0] = a.k[1] = c->at<__nv_bfloat16>(c->L.comp16[1]);
    a.v[0] = a.v[1] = c->at<__nv_bfloat16>(c->L.comp16[2]);
    a.kv_hs[0] = a.kv_hs[1] = rhs; a.n_k[0] = a.n_k[1] = d.R;
    a.kmask[0] = a.kmask[1] = MASK_NONE;
    a.tiles0 = a.tiles_total = a.tiles_per_split = attn_tc_tiles(d.R); a.n_split = 1;
    a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
    a.o32 = c->at<float>(c->L.ocomp); a.o_hs = rhs;
    a.kc = no_sel ? 0 : d.kc; a.cand = c->at<int>(c->L.idx); a.cand_user = sel_idx_out;
    a.guide_only = cf.variant == GSA_VARIANT_NO_COMP_VALUE ? 1 : 0;
    a.rpf = d.rpf; a.n_fixed = cf.num_fixed_frames;
    for (int i = 0; i < cf.num_fixed_frames; ++i) a.fixed[i] = c->fixed[i];
    a.err = err;
    if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
  } else {
    AttnF32Args a;
    memset(&a, 0, sizeof(a));
    a.q = c->at<float>(c->L.comp32[0]); a.q_hs = rhs; a.n_q = d.R; a.q_mask = MASK_NONE;
    a.nseg = 1;
    a.k[0] = a.k[1] = c->at<float>(c->L.comp32[1]);
    a.v[0] = a.v[1] = c->at<float>(c->L.comp32[2]);
    a.kv_hs[0] = a.kv_hs[1] = rhs; a.n_k[0] = a.n_k[1] = d.R;
    a.H = H; a.g = g; a.scale = scale;
    a.o = c->at<float>(c->L.ocomp); a.o_hs = rhs;
    a.kc = d.kc; a.cand = c->at<int>(c->L.idx); a.cand_user = sel_idx_out;
    a.rpf = d.rpf; a.n_fixed = cf.num_fixed_frames;
    for (int i = 0; i < cf.num_fixed_frames; ++i) a.fixed[i] = c->fixed[i];
    if (launch_attn_f32(a, !no_sel, st) != cudaSuccess) return GSA_ERR_CUDA;
  }
  prof.mark(no_sel ? "comp_attn" : cf.variant == GSA_VARIANT_NO_COMP_VALUE ? "comp_guide_topk" : "comp_attn_topk");

  // K3 selection (+ K4 upsample/gate/blend, fused for bf16)
  SelArgs sa;
  sa.q_img = q_img; sa.k_img = k_img; sa.v_img = v_img; sa.k_spec = k_spec; sa.v_spec = v_spec;
  sa.idx = c->at<int>(c->L.idx); sa.o_sel = c->ws + c->L.osel;
  sa.H = H; sa.F = cf.num_frames; sa.R = d.R; sa.rpf = d.rpf; sa.topk = cf.topk; sa.s = cf.pool_s;
  sa.g = g; sa.scale_log2 = scale * LOG2E; sa.n_fixed = cf.num_fixed_frames;
  for (int i = 0; i < cf.num_fixed_frames; ++i) sa.fixed[i] = c->fixed[i];
  sa.err = err;
  EpiArgs ea;
  ea.q_img = q_img; ea.o_sel = c->ws + c->L.osel; ea.o_comp = c->at<float>(c->L.ocomp);
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
    if (launch_sel_fused(sa, ea, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("selection_gate");
  } else {
    if (launch_sel(sa, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("selection");
    if (launch_epilogue(ea, d.fp32, st) != cudaSuccess) return GSA_ERR_CUDA;
    prof.mark("epilogue");
  }

  // K5 special tokens over every token
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
      a.tiles0 = d.spec_tiles0; a.tiles_total = d.spec_tiles_total;
      a.tiles_per_split = d.spec_tps; a.n_split = d.spec_split;
      a.H = H; a.g = g; a.scale_log2 = scale * LOG2E;
      a.o16 = reinterpret_cast<__nv_bfloat16*>(o_spec); a.o_hs = shs;
      a.part_o = c->at<float>(c->L.part_o); a.part_ml = c->at<float>(c->L.part_ml);
      a.err = err;
      if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
      prof.mark("special");
      if (d.spec_split > 1) {
        MergeArgs m;
        m.part_o = a.part_o; m.part_ml = a.part_ml; m.n_split = d.spec_split; m.H = H;
        m.n_q = a.n_q; m.scale_log2 = a.scale_log2; m.o16 = a.o16; m.o32 = nullptr; m.o_hs = shs;
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
  if (!c || limit_us < 1 || limit_us > 1000000) return GSA_ERR_INVALID_ARG;
  DeviceGuard dg(c->device);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
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
