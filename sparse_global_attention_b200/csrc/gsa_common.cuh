// Shared device helpers for the GSA kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gsa {

constexpr int D = 64;            // head dimension (fixed by the layer's configs)
constexpr int KC_MAX = 64;       // largest top-k candidate list per row
constexpr int MAX_FIXED = 16;    // largest number of VGGT fixed-context frames
constexpr float LOG2E = 1.4426950408889634f;

// device error word values (same numbers as GSA_ERR_* in gsa.h)
constexpr int ERR_BOUNDS = 7;
constexpr int ERR_TIMEOUT = 6;

__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// --------------------------------------------------------------------------
// PTX wrappers
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes = 0 zero-fills the slot.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8,f32) += A(16x16,bf16,row) * B(16x8,bf16,col)
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// hardware base-2 exponential (PTX ex2.approx, flush-to-zero)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a [rows][64] bf16
// tile whose chunks are XOR-swizzled by the row's low 3 bits; ldmatrix over
// 8 consecutive rows then touches 8 distinct bank groups.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// --------------------------------------------------------------------------
// token geometry
// --------------------------------------------------------------------------
struct Grid {
  int Hp, Wp, Hv, Wv, ns;   // padded grid, valid grid, special tokens per frame
  __device__ __forceinline__ bool img_valid(int o) const {   // o: index inside one frame's grid
    int y = o / Wp;
    int x = o - y * Wp;
    return y < Hv && x < Wv;
  }
};

// Key-validity modes of a key segment
enum MaskMode : int {
  MASK_NONE = 0,     // keys 0..n-1 all valid
  MASK_IMG = 1,      // keys laid out [F][Hp][Wp]; pads invalid
  MASK_DENSE = 2,    // keys laid out [F][ns + Hp*Wp]; image pads invalid
};

__device__ __forceinline__ bool key_valid(int mode, const Grid& g, long long n) {
  if (mode == MASK_IMG) {
    int per = g.Hp * g.Wp;
    return g.img_valid(static_cast<int>(n % per));
  }
  if (mode == MASK_DENSE) {
    int per = g.ns + g.Hp * g.Wp;
    int o = static_cast<int>(n % per);
    return o < g.ns || g.img_valid(o - g.ns);
  }
  return true;
}

}  // namespace gsa
