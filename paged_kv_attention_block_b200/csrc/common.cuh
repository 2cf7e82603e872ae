// Device helpers: element conversions, async copies, tensor-core fragments.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "plan_format.h"

#define PKV_DEVICE __device__ __forceinline__

namespace pkv {

enum KvKind { KV_BF16 = 0, KV_F16 = 1, KV_E4M3 = 2 };

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

PKV_DEVICE void report(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---- conversions -------------------------------------------------------
PKV_DEVICE float bf16_bits_to_float(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
PKV_DEVICE float f16_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

PKV_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
PKV_DEVICE uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Two E4M3 codes (low byte first) -> f16x2 (exact: every E4M3 value is an f16).
PKV_DEVICE uint32_t e4m3x2_to_f16x2(uint16_t two) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return uint32_t(r.x) | (uint32_t(r.y) << 16);
}

// ---- shared-memory tile layout -------------------------------------------
// A K or V tile is PKV_TILE_KEYS rows of RB = head_dim * elem bytes.  Rows
// wider than 128 B are split into 128-B column slabs, each slab rows x 128 B,
// and 16-byte chunks are XOR-swizzled with address bits 7..9 (the 128-byte
// swizzle pattern), which makes the 8-row ldmatrix / LDS.128 phases of the MMA
// fragment loads bank-conflict free.
template <int RB>
PKV_DEVICE uint32_t tile_offset(int row, int byte) {
  uint32_t lin;
  if constexpr (RB >= 128) {
    lin = uint32_t(byte >> 7) * (PKV_TILE_KEYS * 128) + uint32_t(row) * 128 + uint32_t(byte & 127);
  } else {
    lin = uint32_t(row) * RB + uint32_t(byte);
  }
  return lin ^ (((lin >> 7) & 7) << 4);
}

PKV_DEVICE uint32_t smem_addr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// 16-byte async copy global -> shared; src_bytes = 0 zero-fills.
PKV_DEVICE void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
PKV_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
PKV_DEVICE void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

PKV_DEVICE uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

PKV_DEVICE void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B, m16n8k16, fp32 accumulate; element type bf16 (BF=true) or f16.
template <bool BF>
PKV_DEVICE void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if constexpr (BF) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

PKV_DEVICE float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace pkv
