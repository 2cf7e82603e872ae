// Device helpers: element conversions, async copies, tensor-core fragments.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "plan_format.h"

#define PKV_DEVICE __device__ __forceinline__

namespace pkv {

enum KvKind { KV_BF16 = 0, KV_F16 = 1, KV_E4M3 = 2, KV_NVFP4 = 3 };

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

// Integer dequantisation into f16 bit patterns, for the decode tiles where conversion
// instructions would be the bottleneck.  Placing a code's exponent and mantissa bits into the
// low bits of the f16 exponent and the top of its mantissa (sign to bit 15) yields the code's
// value times a fixed power of two, subnormals included: 2^-8 for E4M3 (exponent bias 15
// against 7), 2^-14 for E2M1 (bias 15 against 1).  NaN codes come out finite.
//
// E4M3 codes in bytes 0 and 2 of w -> f16x2 (byte 0, byte 2) * 2^-8; bytes 1, 3 are ignored.
PKV_DEVICE uint32_t e4m3_b02_f16x2(uint32_t w) { return ((w << 7) & 0x3F803F80u) | ((w << 8) & 0x80008000u); }
// E4M3 codes in bytes 1 and 3 of w -> f16x2 (byte 1, byte 3) * 2^-8; bytes 0, 2 are ignored.
PKV_DEVICE uint32_t e4m3_b13_f16x2(uint32_t w) { return ((w >> 1) & 0x3F803F80u) | (w & 0x80008000u); }
// E2M1 codes in nibbles I and I + 4 of w -> f16x2 (nibble I, nibble I+4) * 2^-14.
template <int I>
PKV_DEVICE uint32_t e2m1_pair_f16x2(uint32_t w) {
  const uint32_t x = w << (12 - 4 * I);  // nibble I -> bits 12..15, nibble I+4 -> bits 28..31
  return ((x >> 3) & 0x0E000E00u) | (x & 0x80008000u);
}
// All four nibble pairs (i, i + 4) of w at once, p[i] = e2m1_pair_f16x2<i>(w), in 13 integer
// operations instead of 15: in every byte of the even and of the odd nibbles one multiply-add
// (n + 7 (n & 8)) moves the sign from bit 3 to bit 6, leaving the magnitude in bits 0-2 with three
// zero bits between (the f16 pattern); after a shift by one, byte permutes place the bytes.
PKV_DEVICE void e2m1_word_f16x2(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t es = (e + 7u * (e & 0x08080808u)) << 1, os = (o + 7u * (o & 0x08080808u)) << 1;
  p[0] = __byte_perm(es, 0, 0x2404);  // nibbles 0, 4 (bytes 0, 2 of the even nibbles)
  p[2] = __byte_perm(es, 0, 0x3414);  // nibbles 2, 6
  p[1] = __byte_perm(os, 0, 0x2404);  // nibbles 1, 5
  p[3] = __byte_perm(os, 0, 0x3414);  // nibbles 3, 7
}
constexpr uint32_t kF16Pow2_15x2 = 0x78007800u;  // f16x2 (2^15, 2^15)
// f16x2 product, round to nearest (exact for the scaled E2M1 and E4M3 values multiplied here).
PKV_DEVICE uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ---- shared-memory tile layout -------------------------------------------
// A K or V tile is TK rows (keys) of RB = head_dim * elem bytes.  Rows
// wider than 128 B are split into 128-B column slabs, each slab rows x 128 B,
// and 16-byte chunks are XOR-swizzled with address bits 7..9 (the 128-byte
// swizzle pattern), which makes the 8-row ldmatrix / LDS.128 phases of the MMA
// fragment loads bank-conflict free.
// SLAB is the distance between column slabs (TK * 128 when a tile's slabs are
// adjacent; larger when K and V slabs interleave).
template <int RB, int TK = PKV_TILE_KEYS, int SLAB = TK * 128>
PKV_DEVICE uint32_t tile_offset(int row, int byte) {
  uint32_t lin;
  if constexpr (RB >= 128) {
    lin = uint32_t(byte >> 7) * SLAB + uint32_t(row) * 128 + uint32_t(byte & 127);
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

PKV_DEVICE uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

PKV_DEVICE uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

PKV_DEVICE void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
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

// First key a causal row at position pos may see under a limited attention
// window (keys pos - window < t <= pos); 0 without a window or for rows that
// have no position (non-causal, padding).
PKV_DEVICE int window_start(int window, int pos) { return (window > 0 && pos >= 0) ? pos + 1 - window : 0; }

// ---- programmatic dependent launch -------------------------------------------
// A grid launched with programmatic stream serialization may start before the
// kernel ahead of it on the stream has finished.  pdl_wait blocks until that
// kernel has completed and its memory operations are visible; pdl_trigger lets
// this grid's dependent be scheduled before this grid finishes (each CTA
// triggers; a CTA that exits counts as triggered).
PKV_DEVICE void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
PKV_DEVICE void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- packed float pairs (sm_100 f32x2 arithmetic) and an FMA-pipe exp2 -----

PKV_DEVICE float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 pa, pb, pc, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n mov.b64 pc, {%6, %7};\n"
      " fma.rn.f32x2 pd, pa, pb, pc;\n mov.b64 {%0, %1}, pd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
PKV_DEVICE float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
      " add.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x for a pair, on the FMA pipe (the softmax is bound by the exp unit, so a
// share of its exponentials is computed here instead).  Range reduction: adding
// 1.5 * 2^23 rounds x to the nearest integer j, held in the low mantissa bits of
// the sum; f = x - j lies in [-1/2, 1/2].  2^f is a cubic fitted to 2^f on
// [-1/2, 1/2] by weighted least squares iterated towards equal relative error
// (csrc/exp2_poly_fit.py); its largest relative error is 7.5e-5, below the
// rounding of P to 16 bits.  2^j is added to the exponent field: the sum's bits
// are 0x4B400000 + j, and (0x4B400000 << 23) is 0 modulo 2^32, so shifting the
// sum's bits left by 23 gives j << 23.  x is clamped at -125, where the result
// is still a normal number; exact values below that are < 2^-125 and do not
// matter next to the row maximum's 2^0.
constexpr float kExp2C0 = 0.99992806f, kExp2C1 = 0.69326097f, kExp2C2 = 0.24261113f, kExp2C3 = 0.055171665f;
constexpr float kRoundShift = 12582912.f;  // 1.5 * 2^23
PKV_DEVICE float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = fadd2(x, make_float2(kRoundShift, kRoundShift));
  const float2 j = fadd2(t, make_float2(-kRoundShift, -kRoundShift));
  const float2 f = ffma2(j, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = ffma2(p, f, make_float2(kExp2C1, kExp2C1));
  p = ffma2(p, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace pkv

// ---- mbarriers, TMA, warp-level matrix moves (sm_90+ PTX) -----------------
namespace pkv {

PKV_DEVICE void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
PKV_DEVICE void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
PKV_DEVICE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

PKV_DEVICE void mbar_arrive(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
PKV_DEVICE void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
PKV_DEVICE bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity: false once `limit` SM cycles
// have passed (by default 4e9: 2.0 s at 1965 MHz, about 3 s at 1.3 GHz); the
// caller records an error and stops waiting.  The deadline uses the SM-local
// cycle counter, which is cheap to read.
PKV_DEVICE bool mbar_wait(uint32_t bar, uint32_t parity, long long limit = PKV_DEFAULT_WAIT_CYCLES) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit) return false;
  }
}
// The same wait with the limit read from shared memory (where a kernel keeps its per-launch
// limit), only once the first try has failed: the hot path holds no register for it.
PKV_DEVICE bool mbar_wait(uint32_t bar, uint32_t parity, const long long* limit_smem) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long limit = *static_cast<const volatile long long*>(limit_smem);
  return mbar_wait(bar, parity, limit);
}

// 1-D bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global into
// shared memory, completion counted on `bar` (no multicast).
PKV_DEVICE void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// 5-D tiled TMA load into shared memory, completion counted on `bar` (no multicast).
PKV_DEVICE void tma_load_5d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], "
      "[%2];\n" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

PKV_DEVICE void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose an 8x8 matrix of 16-bit elements held one row pair per thread.
PKV_DEVICE uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

PKV_DEVICE void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace pkv

namespace pkv {
// Merge element of a row whose n partial states sit at o_of(i), lse_of(i)
// (normalised o, natural-log lse; lse = -inf marks an empty part):
//   M = max lse_i, w_i = exp(lse_i - M), o = sum w_i o_i / sum w_i, lse = M + ln sum w_i.
template <typename LseOf, typename OOf>
PKV_DEVICE void merge_elem(int n, LseOf lse_of, OOf o_of, float& o, float& lse) {
  float M = -INFINITY;
  for (int i = 0; i < n; ++i) M = fmaxf(M, lse_of(i));
  if (M == -INFINITY) {
    o = 0.f;
    lse = -INFINITY;
    return;
  }
  float num = 0.f, den = 0.f;
  for (int i = 0; i < n; ++i) {
    const float li = lse_of(i);
    if (li == -INFINITY) continue;
    const float w = expf(li - M);
    den += w;
    num = fmaf(w, o_of(i), num);
  }
  o = num / den;
  lse = M + logf(den);
}

PKV_DEVICE void store_any(void* out, int dtype, int64_t idx, float v) {
  if (dtype == 0) static_cast<float*>(out)[idx] = v;
  else if (dtype == 1) static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(out)[idx] = __float2half_rn(v);
}
}  // namespace pkv
