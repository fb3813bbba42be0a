// tcgen05 / TMEM helpers and the fp16 dequantization shared by the tensor-core
// matmul kernels (sm_100a only).
#pragma once

#include "common.cuh"

namespace aq {
namespace qmm {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
AQ_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
AQ_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

AQ_DEVICE void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate)
AQ_DEVICE void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

AQ_DEVICE void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
AQ_DEVICE void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

AQ_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
AQ_DEVICE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row atoms of
// 1024 bytes (stride byte offset 1024), descriptor version 1 (sm_100).
AQ_DEVICE uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);      // start address
  d |= static_cast<uint64_t>(1u) << 16;                        // leading byte offset (unused with swizzle)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                        // version
  d |= static_cast<uint64_t>(2u) << 61;                        // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f16 with A = B = fp16 (format 0), D = f32
// (format 1), both K-major, M = 128, N = bn.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int bn) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(bn >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Dequantization of one 32-code chunk into 16 TMEM columns of fp16 pairs.
//
// Bits 2, 4 and 8: codes become exact fp16 values 1024 + q by OR-ing them into
// the mantissa of 1024.0 (one logic op or byte permute per two codes), then
// q = (1024 + q) - 1024 and w = q*scale + bias with packed fp16 arithmetic:
// one rounding, w = fp16_rn(q*scale + bias).  The two codes of a pair are
// (j, j+4) of a word for 4-bit and (j, j+8) for 2-bit, so the chunk's K order
// is interleaved in blocks of 8 (resp. 16) elements; the activation pre-pass
// writes x16 in the same order (kx_perm below), which leaves the product
// unchanged.  8-bit pairs are adjacent bytes (natural order).  3-bit codes go
// through fp32 (exact q via the mantissa trick, one fp32 FMA, then RNE to fp16).
// ---------------------------------------------------------------------------
template <int BITS>
AQ_DEVICE void dequant_chunk_f16(const uint32_t (&w)[BITS], uint16_t sc_bits, uint16_t bi_bits,
                                 uint32_t (&cols)[16]) {
  if constexpr (BITS == 4 || BITS == 2) {
    // Pair j of a word holds codes j and j + PER_WORD.  Pairs 0..PER_WORD/2-1
    // are masked in place from the word (codes at bit offset BITS*j inside each
    // 16-bit half) and the rest from the word shifted right by 8, so one shift
    // per word suffices.  A code at offset BITS*j' inside the half reads as
    // 1024 + q*2^(BITS*j'); q = h*2^-(BITS*j') - 1024*2^-(BITS*j') exactly.
    constexpr int PER_WORD = 32 / BITS / 2;  // pairs per word: 4 (4-bit) or 8 (2-bit)
    constexpr int IN_BYTE = PER_WORD / 2;    // pairs per shifted copy: 2 or 4
    constexpr uint32_t LO = (1u << BITS) - 1u;
    const __half2 s2 = __half2half2(__ushort_as_half(sc_bits));
    const __half2 b2 = __half2half2(__ushort_as_half(bi_bits));
    const uint32_t magic = 0x64006400u;
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const uint32_t src[2] = {w[i], w[i] >> 8};
      static_for<0, PER_WORD>([&](auto J) {
        constexpr int j = J.value;
        constexpr int jj = j % IN_BYTE;  // position inside the byte
        constexpr uint32_t MASK = (LO | (LO << 16)) << (BITS * jj);
        const uint32_t v = lop3_and_or<MASK>(src[j / IN_BYTE], magic);
        __half2 h = *reinterpret_cast<const __half2 *>(&v);
        if constexpr (jj == 0) {
          h = __hsub2(h, __half2half2(__ushort_as_half(0x6400)));  // - 1024
        } else {
          // h * 2^-(BITS*jj) - 1024 * 2^-(BITS*jj): both constants exact in fp16
          constexpr unsigned short INV = static_cast<unsigned short>((15 - BITS * jj) << 10);
          constexpr unsigned short OFF = static_cast<unsigned short>(0x8000u | ((25 - BITS * jj) << 10));
          h = __hfma2(h, __half2half2(__ushort_as_half(INV)), __half2half2(__ushort_as_half(OFF)));
        }
        h = __hfma2(h, s2, b2);
        cols[PER_WORD * i + j] = *reinterpret_cast<uint32_t *>(&h);
      });
    }
  } else if constexpr (BITS == 8) {
    const __half2 s2 = __half2half2(__ushort_as_half(sc_bits));
    const __half2 b2 = __half2half2(__ushort_as_half(bi_bits));
    const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));
    const uint32_t magic = 0x64646464u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // bytes of the result: [code0, 0x64, code1, 0x64] -> (1024 + code0, 1024 + code1)
      const uint32_t v0 = __byte_perm(w[i], magic, 0x5140u);
      const uint32_t v1 = __byte_perm(w[i], magic, 0x5342u);
      __half2 h0 = *reinterpret_cast<const __half2 *>(&v0);
      __half2 h1 = *reinterpret_cast<const __half2 *>(&v1);
      h0 = __hfma2(__hsub2(h0, k1024), s2, b2);
      h1 = __hfma2(__hsub2(h1, k1024), s2, b2);
      cols[2 * i] = *reinterpret_cast<uint32_t *>(&h0);
      cols[2 * i + 1] = *reinterpret_cast<uint32_t *>(&h1);
    }
  } else {
    const float scf = half_bits_to_float(sc_bits), bif = half_bits_to_float(bi_bits);
    static_for<0, 16>([&](auto P) {
      constexpr int j = 2 * P.value;
      const float2 f = make_float2(__uint_as_float(extract_magic<BITS, j>(w)),
                                   __uint_as_float(extract_magic<BITS, j + 1>(w)));
      const float2 u = fadd2(f, make_float2(-1.0f, -1.0f));  // q * 2^(p-23), exact
      constexpr float f0 = field_factor(BITS, j), f1 = field_factor(BITS, j + 1);
      const float2 v = ffma2(u, make_float2(scf * f0, scf * f1), make_float2(bif, bif));  // fp32_rn(q*s + b)
      __half2 h2 = __floats2half2_rn(v.x, v.y);
      cols[P.value] = *reinterpret_cast<uint32_t *>(&h2);
    });
  }
}

// ---------------------------------------------------------------------------
// Block-scaled formats (prefill): one 32-code chunk into 16 TMEM columns of
// fp16 pairs, each value scaled by a power of two 2^-B of its W row (B from
// the row's largest scale, so every value is an exact fp16 for groups within
// 2^22 of the row's largest; the epilogue multiplies by 2^B).
//
// E2M1 code m (sign in bit 3) as fp16 bits ((m & 7) << 9 | (m & 8) << 12) is
// the code's value times 2^-14 (exponent field and mantissa bit line up; the
// one subnormal code, 0.5, becomes fp16's subnormal 2^-15); E4M3 byte b as
// ((b & 0x7F) << 7 | (b & 0x80) << 8) is its value times 2^-8.  The chunk is
// then one packed fp16 multiply by the group's factor (exact: a power of two,
// or an E4M3 value for nvfp4), in the pair order of the affine 4-bit and
// 8-bit paths (so the same x16 interleave serves).
// ---------------------------------------------------------------------------
// E2M1 chunk (mxfp4, nvfp4): f_lo scales words 0-1 (codes 0..15), f_hi words
// 2-3 (codes 16..31): the same factor for mxfp4, the two 16-code groups' for
// nvfp4.  Each factor is a value of at most 4 significant bits.
AQ_DEVICE void dequant_chunk_e2m1(const uint32_t (&w)[4], __half2 f_lo, __half2 f_hi, uint32_t (&cols)[16]) {
  const __half2 two14 = __half2half2(__ushort_as_half(0x7400));  // 2^14: the bits above read as value * 2^-14
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 f = i < 2 ? f_lo : f_hi;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t v = (w[i] >> (4 * j)) & 0x000F000Fu;  // codes j and j + 4 of the word
      const uint32_t h = ((v & 0x00070007u) << 9) | ((v & 0x00080008u) << 12);
      __half2 x = __hmul2(*reinterpret_cast<const __half2 *>(&h), two14);  // the E2M1 values, exact
      x = __hmul2(x, f);
      cols[4 * i + j] = *reinterpret_cast<uint32_t *>(&x);
    }
  }
}
// E4M3 chunk (mxfp8; four codes per word, natural order): f = the group's
// factor times 2^8 (the bits above read as value * 2^-8).
AQ_DEVICE void dequant_chunk_e4m3(const uint32_t (&w)[8], __half2 f, uint32_t (&cols)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t v = w[i] >> (16 * j);
      const uint32_t b0 = v & 0xFFu, b1 = (v >> 8) & 0xFFu;
      const uint32_t h = (((b0 & 0x7Fu) << 7) | ((b0 & 0x80u) << 8)) |
                         ((((b1 & 0x7Fu) << 7) | ((b1 & 0x80u) << 8)) << 16);
      __half2 x = __hmul2(*reinterpret_cast<const __half2 *>(&h), f);
      cols[2 * i + j] = *reinterpret_cast<uint32_t *>(&x);
    }
  }
}
// 2^e as an fp32 (exact for e in [-149, 127]; 0 below)
AQ_DEVICE float pow2f_exact(int e) {
  if (e >= -126) return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  if (e >= -149) return __uint_as_float(1u << (e + 149));
  return 0.0f;
}
// value of an E4M3 byte (exact in fp32)
AQ_DEVICE float e4m3_value(uint32_t b) {
  const uint16_t h = static_cast<uint16_t>(((b & 0x7Fu) << 7) | ((b & 0x80u) << 8));  // value * 2^-8
  return __half2float(__ushort_as_half(h)) * 256.0f;
}

// K order of x16 inside each block of 8 (4-bit) or 16 (2-bit) elements: slot t
// holds element kx_perm(t) of the block, matching the pairs of dequant_chunk_f16.
__host__ __device__ constexpr int kx_block(int bits) { return bits == 4 ? 8 : bits == 2 ? 16 : 1; }
__host__ __device__ constexpr int kx_perm(int bits, int t) {
  return kx_block(bits) == 1 ? t : (t % 2) * (kx_block(bits) / 2) + t / 2;
}

}  // namespace qmm
}  // namespace aq
