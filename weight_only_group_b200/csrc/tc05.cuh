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

// K order of x16 inside each block of 8 (4-bit) or 16 (2-bit) elements: slot t
// holds element kx_perm(t) of the block, matching the pairs of dequant_chunk_f16.
__host__ __device__ constexpr int kx_block(int bits) { return bits == 4 ? 8 : bits == 2 ? 16 : 1; }
__host__ __device__ constexpr int kx_perm(int bits, int t) {
  return kx_block(bits) == 1 ? t : (t % 2) * (kx_block(bits) / 2) + t / 2;
}

}  // namespace qmm
}  // namespace aq
