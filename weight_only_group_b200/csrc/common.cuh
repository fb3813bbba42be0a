// Shared device helpers of the CUDA path (sm_100a only).  Nothing here is
// shared with, or derived from, the CPU oracle.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/aq.h"

#define AQ_DEVICE __device__ __forceinline__

namespace aq {

// One matmul of a sequence launch (device pointers; bf16 x [M, K], y [M, N]).
struct SeqCall {
  const uint16_t *x;
  const uint32_t *packed;
  const uint16_t *scales, *biases;
  uint16_t *y;
  int64_t N, K;
};


// Bits of the device-side fault word (defined next to the only kernel with
// waits): set, never trapped, when a bounded wait gives up.
enum : uint32_t {
  kFaultMmaWait = 1u << 0,      // MMA issuer gave up waiting for operands
  kFaultProducerWait = 1u << 1, // TMA producer gave up waiting for a free stage
  kFaultDequantWait = 1u << 2,  // dequant warps gave up waiting for packed data / a free A stage
  kFaultEpilogueWait = 1u << 3, // epilogue gave up waiting for the accumulator
  kFaultQmvWait = 1u << 4,      // QMV gave up waiting for a weight stage
  kFaultBadIndex = 1u << 5,     // an embedding id outside [0, V): that output row was zeroed
};

// Upper bound of any spin on an mbarrier, in SM clock cycles (~1 s at 2 GHz).
constexpr long long kWaitCycles = 2000000000LL;

// ---------------------------------------------------------------------------
// Loads
// ---------------------------------------------------------------------------
AQ_DEVICE uint4 ldg_stream16(const void *p) {  // read-once stream: skip L1
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
AQ_DEVICE uint4 ldg_nc16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
AQ_DEVICE uint2 ldg_nc8(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
AQ_DEVICE uint32_t ldg_nc4(const void *p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
AQ_DEVICE uint16_t ldg_nc2(const void *p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

AQ_DEVICE float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }
AQ_DEVICE float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

AQ_DEVICE uint32_t smem_u32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// Packed fp32x2 arithmetic (sm_100 builtins): two FMAs / adds per instruction.
AQ_DEVICE float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
AQ_DEVICE float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy helpers (shared memory addresses as 32-bit)
// ---------------------------------------------------------------------------
AQ_DEVICE void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
AQ_DEVICE void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
AQ_DEVICE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
AQ_DEVICE bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true once the phase with the given parity has completed; false
// on timeout (the fault bit is OR-ed into *fault and *abort_flag is raised) or
// when another thread of the CTA has already raised *abort_flag.
// `limit` is the number of SM clock cycles after which the wait gives up.
AQ_DEVICE bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *fault,
                         uint32_t fault_bit, long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      atomicOr(fault, fault_bit);
      *abort_flag = 1;
      return false;
    }
  }
}
// Bounded wait used while shutting down after an abort: it ignores the abort
// flag (the point is to let copies or MMAs already issued complete before the
// CTA exits or frees what they write to) and gives up after kWaitCycles.
AQ_DEVICE bool mbar_drain(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}
AQ_DEVICE void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte aligned, size % 16 == 0).
AQ_DEVICE void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 2-D tiled TMA load global -> this CTA's shared memory, completing on an
// mbarrier; c0 is the innermost coordinate, c0 * element size % 16 == 0.
AQ_DEVICE void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Code extraction into "magic" floats.
//
// A code field of `bits` bits is moved, by a rotation of its 32-bit word by a
// multiple of 8, to a position p inside the fp32 mantissa and OR-ed with the
// exponent of 1.0, giving the float f = 1 + q * 2^(p-23) exactly.  p is chosen
// in [16-bits, 23-bits] so the field's top bit lies at 15..22.  The consumer
// recovers q*x as x*2^(23-p)*f - x*2^(23-p); the 2^(23-p) factor is folded
// into pre-scaled activations, so all products of one chunk accumulate in one
// register.  Rotations by multiples of 8 are shared by the fields of a word.
// ---------------------------------------------------------------------------
constexpr uint32_t kOne = 0x3F800000u;

struct FieldPlace {
  int word;      // word of the chunk holding the field's first bit
  int off;       // bit offset of the field in that word
  int rot;       // left rotation applied (0/8/16/24), or -1 if the field straddles two words
  int p;         // mantissa bit where the field lands
};

__host__ __device__ constexpr int field_pmin(int bits) { return 16 - bits; }
__host__ __device__ constexpr int field_pmax(int bits) { return 23 - bits; }

__host__ __device__ constexpr FieldPlace field_place(int bits, int j) {
  const int bp = j * bits, word = bp / 32, off = bp % 32;
  if (off + bits > 32) return FieldPlace{word, off, -1, field_pmax(bits)};
  if (bits == 8) return FieldPlace{word, off, 0, 8};  // byte permute, see extract_magic
  for (int r = 0; r < 32; r += 8) {
    const int p = (off + r) % 32;
    if (p >= field_pmin(bits) && p <= field_pmax(bits)) return FieldPlace{word, off, r, p};
  }
  return FieldPlace{word, off, -2, 0};  // unreachable for bits in {2,3,4}
}

// 2^(23 - p) for code j of a 32-code chunk.
__host__ __device__ constexpr float field_factor(int bits, int j) {
  const int e = 23 - field_place(bits, j).p;
  float f = 1.0f;
  for (int i = 0; i < e; ++i) f *= 2.0f;
  return f;
}

// (a & b) | c as one three-input logic operation (truth table 0xEA).
template <uint32_t B>
AQ_DEVICE uint32_t lop3_and_or(uint32_t a, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(B), "r"(c));
  return d;
}

// Magic float bits for code J (0..31) of a chunk held in w[0..BITS-1].
template <int BITS, int J>
AQ_DEVICE uint32_t extract_magic(const uint32_t (&w)[BITS]) {
  constexpr FieldPlace fp = field_place(BITS, J);
  constexpr uint32_t mask = (1u << BITS) - 1u;
  if constexpr (BITS == 8) {
    // bytes of the result: [0x00, code, 0x80, 0x3F] -> 1 + code * 2^-15
    constexpr uint32_t sel = 0x7604u | (uint32_t(fp.off / 8) << 4);
    return __byte_perm(w[fp.word], kOne, sel);
  } else if constexpr (fp.rot < 0) {
    const uint32_t v = __funnelshift_r(w[fp.word], w[fp.word + 1], fp.off);
    return lop3_and_or<(mask << fp.p)>(v << fp.p, kOne);
  } else {
    const uint32_t v = fp.rot ? __funnelshift_l(w[fp.word], w[fp.word], fp.rot) : w[fp.word];
    return lop3_and_or<(mask << fp.p)>(v, kOne);
  }
}

// Code J as an exact small integer (for the quantize/dequantize kernels).
template <int BITS, int J>
AQ_DEVICE uint32_t extract_code(const uint32_t (&w)[BITS]) {
  constexpr int bp = J * BITS, word = bp / 32, off = bp % 32;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  if constexpr (off + BITS <= 32) {
    return (w[word] >> off) & mask;
  } else {
    return __funnelshift_r(w[word], w[word + 1], off) & mask;
  }
}

// ---------------------------------------------------------------------------
// Host: encoded 2-D TMA descriptors, cached per thread.  A descriptor is a pure
// function of its arguments (base address, element type, sizes, strides, box,
// swizzle), so a hit returns exactly what encoding again would; the cache only
// saves the driver call on repeated calls with the same operands.
// ---------------------------------------------------------------------------
struct TmapKey {
  const void *base;
  uint64_t dim0, dim1, stride1;
  uint32_t box0, box1, dtype, swizzle;
  bool operator==(const TmapKey &o) const {
    return base == o.base && dim0 == o.dim0 && dim1 == o.dim1 && stride1 == o.stride1 && box0 == o.box0 &&
           box1 == o.box1 && dtype == o.dtype && swizzle == o.swizzle;
  }
};

template <class EncodeFn>
inline bool encode_2d_cached(EncodeFn fn, CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                             uint64_t dim0, uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                             CUtensorMapSwizzle swizzle) {
  constexpr int kSlots = 64;
  struct Slot {
    TmapKey key;
    CUtensorMap map;
    bool used;
  };
  static thread_local Slot slots[kSlots] = {};
  const TmapKey key{base, dim0, dim1, stride1_bytes, box0, box1, static_cast<uint32_t>(dtype),
                    static_cast<uint32_t>(swizzle)};
  uint64_t h = reinterpret_cast<uintptr_t>(base) ^ (dim0 * 0x9E3779B97F4A7C15ull) ^ (dim1 << 17) ^ (box0 << 7) ^
               (uint64_t(box1) << 29) ^ (uint64_t(dtype) << 3) ^ (uint64_t(swizzle) << 11);
  h ^= h >> 29;
  Slot &sl = slots[h % kSlots];
  if (sl.used && sl.key == key) {
    *map = sl.map;
    return true;
  }
  cuuint64_t dims[2] = {dim0, dim1};
  cuuint64_t strides[1] = {stride1_bytes};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t estr[2] = {1, 1};
  if (fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  sl.key = key;
  sl.map = *map;
  sl.used = true;
  return true;
}

template <int N>
struct Int {
  static constexpr int value = N;
};

template <int Begin, int End, class F>
AQ_DEVICE void static_for(F &&f) {
  if constexpr (Begin < End) {
    f(Int<Begin>{});
    static_for<Begin + 1, End>(f);
  }
}

}  // namespace aq
