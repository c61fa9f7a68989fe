// Special-token attention without any device allocation.
//
// Some callers cannot call cudaMalloc: a host program or serving engine that
// reserves all device memory up front and hands a kernel only its inputs and
// outputs, or a latency-critical loop where an allocation's implicit
// synchronisation is not acceptable.  For them this entry point runs the
// split-key special-token attention with its per-split partial results
// (running max, sum and unnormalised output per row and split) in one
// file-scope device array of fixed size instead of a context workspace.
//
// The array's name is only a host-side stand-in; its device address is taken
// with cudaGetSymbolAddress once per device, on the first call made with that
// device current, and cached.  Make that first call before any stream capture.
// Every call shares the array and finds the previous call's contents in it;
// the split kernel writes every partial entry that the merge reads, so nothing
// needs clearing.  The array's first word is the device status word of these
// calls: a kernel whose bounded wait runs out, or whose index check fails,
// records its code there.  It starts at zero (static device memory is zero at
// load), stays set until gsa_special_attention_noalloc_status reads and
// clears it, and while it is set later calls stop early (as a context's
// kernels do while its error word is set).  Calls that overlap on the GPU race
// on the array: serialise them (for example, one stream).
#include <mutex>
#include <string.h>

#include "../../include/gsa.h"
#include "gsa_kernels.h"

using namespace gsa;

namespace {

constexpr size_t STATUS_BYTES = 256;
static __device__ __align__(256) uint8_t g_noalloc_scratch[GSA_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void* g_addr[MAX_DEVICES] = {};

// device address of the scratch array on the current device (set up once)
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return GSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GSA_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return GSA_OK;
}

}  // namespace

namespace gsa {
// the status word of the allocation-free calls on the current device
int noalloc_status_word(int** out) {
  void* base = nullptr;
  const int rc = scratch_address(&base);
  if (rc != GSA_OK) return rc;
  *out = static_cast<int*>(base);
  return GSA_OK;
}
}  // namespace gsa

extern "C" int gsa_special_attention_noalloc_status(void* stream) {
  int* word = nullptr;
  int rc = noalloc_status_word(&word);
  if (rc != GSA_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GSA_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GSA_ERR_CUDA;
  if (code != 0 && cudaMemset(word, 0, sizeof(int)) != cudaSuccess) return GSA_ERR_CUDA;
  return code;
}

extern "C" int gsa_special_attention_noalloc(const void* q_spec, const void* k_spec, const void* v_spec,
                                             const void* k_img, const void* v_img, void* o_spec,
                                             int num_heads, int num_frames, int num_special, int grid_h,
                                             int grid_w, int pad_h, int pad_w, float softmax_scale,
                                             void* stream) {
  if (!q_spec || !k_spec || !v_spec || !k_img || !v_img || !o_spec) return GSA_ERR_INVALID_ARG;
  if (num_heads < 1 || num_frames < 1 || num_special < 1 || grid_h < 1 || grid_w < 1 ||
      pad_h < grid_h || pad_w < grid_w || !(softmax_scale >= 0.f))
    return GSA_ERR_INVALID_ARG;
  const long long M = static_cast<long long>(num_frames) * num_special;      // special rows per head
  const long long N = static_cast<long long>(num_frames) * pad_h * pad_w;    // image slots per head
  if (M * num_heads >= (1LL << 31) || N * num_heads >= (1LL << 31)) return GSA_ERR_UNSUPPORTED;

  // same split rule as the context path: enough CTAs to fill the GPU
  const int tiles0 = attn_tc_tiles(M);
  const int tiles_total = tiles0 + attn_tc_tiles(N);
  int tps = 0, n_split = 0;
  attn_tc_split(num_heads, M, tiles_total, &tps, &n_split);

  // the partials must fit the static array: otherwise reject, allocate nothing
  const size_t rows = static_cast<size_t>(n_split) * num_heads * M;
  const size_t need = STATUS_BYTES + rows * D * 4 + rows * 2 * 4;
  if (need > GSA_NOALLOC_SCRATCH_BYTES) return GSA_ERR_UNSUPPORTED;

  void* base = nullptr;
  int rc = scratch_address(&base);
  if (rc != GSA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(base);
  int* err = reinterpret_cast<int*>(b);
  float* part_o = reinterpret_cast<float*>(b + STATUS_BYTES);
  float* part_ml = part_o + rows * D;

  const float scale = softmax_scale > 0.f ? softmax_scale : 0.125f;   // 1/sqrt(64)
  Grid g;
  g.Hp = pad_h; g.Wp = pad_w; g.Hv = grid_h; g.Wv = grid_w; g.ns = num_special;
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = static_cast<const __nv_bfloat16*>(q_spec); a.q_hs = M * D; a.n_q = static_cast<int>(M);
  a.q_mask = MASK_NONE;
  a.nseg = 2;
  a.k[0] = static_cast<const __nv_bfloat16*>(k_spec); a.v[0] = static_cast<const __nv_bfloat16*>(v_spec);
  a.kv_hs[0] = M * D; a.n_k[0] = static_cast<int>(M); a.kmask[0] = MASK_NONE;
  a.k[1] = static_cast<const __nv_bfloat16*>(k_img); a.v[1] = static_cast<const __nv_bfloat16*>(v_img);
  a.kv_hs[1] = N * D; a.n_k[1] = static_cast<int>(N);
  a.kmask[1] = (pad_h != grid_h || pad_w != grid_w) ? MASK_IMG : MASK_NONE;
  a.tiles0 = tiles0; a.tiles_total = tiles_total; a.tiles_per_split = tps; a.n_split = n_split;
  a.H = num_heads; a.g = g; a.scale_log2 = scale * LOG2E;
  a.o16 = static_cast<__nv_bfloat16*>(o_spec); a.o_hs = M * D;
  a.part_o = part_o; a.part_ml = part_ml;
  a.err = err;
  if (launch_attn_tc(a, st) != cudaSuccess) return GSA_ERR_CUDA;
  if (n_split > 1) {
    MergeArgs m;
    m.lse = nullptr;
    m.part_o = part_o; m.part_ml = part_ml; m.n_split = n_split; m.H = num_heads;
    m.n_q = static_cast<int>(M); m.scale_log2 = a.scale_log2; m.o16 = a.o16; m.o32 = nullptr; m.o_hs = M * D;
    if (launch_merge(m, st) != cudaSuccess) return GSA_ERR_CUDA;
  }
  return GSA_OK;
}
