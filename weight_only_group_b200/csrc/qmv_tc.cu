// QMV on the tensor cores: y[M,N] = x[M,K] . dequant(W)^T for decode, M = 1..8
// activation rows, W never materialised.
//
// Method: metalworking "MLX Quantization", section "Mechanics" (QMV streams
// each weight once per decode step and dequantizes on the fly; multi-token
// decode, M = 3..6, must still read W once) and anllm "Tutorial 10:
// Quantization", section 5 (y = x @ W^T on the packed weights).  Per group g of
// a row: y += s_g * sum_k q_k x_k + b_g * sum_k x_k.
//
// Why the tensor cores on a bandwidth-bound product: on the CUDA cores, code
// extraction plus one FMA per weight and activation reads from shared memory
// took longer than streaming the weights at B200's HBM rate (measured: the
// arithmetic of a 14336x4096 4-bit call alone ran 1.4x longer than its copies
// alone).  Here the integer tensor cores (mma.sync m16n8k32, u8 x s8, int32
// accumulate) do the multiply-adds and the CUDA cores only unpack codes
// into bytes: three logic ops per 8 codes at 4 bits, none at 8 bits.  mma.sync
// rather than tcgen05: its B operand sits in registers, so the per-lane zero
// masking below costs one select per group, while a shared-memory B operand
// would need eight zero-padded copies of x.
//
// Layout of the arithmetic:
//  * MMA rows = 16 rows of W (a tile); MMA K = 32 codes of one group, as
//    bytes (codes are permuted inside the group so each lane's A registers
//    come from its own packed words; the activations are staged in the same
//    permutation).
//  * Activations: per group, x_int = rint(x * 2^e) with 2^e the power of two
//    that puts the group's largest |x| in [2^13, 2^14), so |x_int| <= 2^14
//    and the rounding error is at most 2^-14 of the group's largest |x|.
//    x_int = 256 * hi + lo with signed digits, lo in [-128, 127] and hi in
//    [-64, 64]; u8 codes x s8 digits give sum q*lo and sum q*hi exactly in
//    int32.
//  * MMA columns (affine codes): column n = 2p + d holds digit plane d of
//    position p, so one MMA per A tile yields both digit sums.  With MP = M
//    rounded up to a power of two, the four positions of an MMA are tokens
//    p / (4/MP) and group slots p % (4/MP) (MP <= 4), or four tokens (MP = 8,
//    two MMAs per A tile).  A lane reads the real activations only while the
//    current group's slot is its column's slot, and zeros otherwise, so one
//    accumulator holds 4/MP groups side by side and is folded once per 4/MP
//    groups:
//        y += s * 2^-e * (256 * D_hi + D_lo) + b * sum x
//    (The block-scaled formats keep one digit plane per MMA, columns = token x
//    group slot, 8/MP slots per fold.)
//  * Streaming: a producer warp copies (16-row tile, K chunk) stages into a
//    shared-memory ring: three 2-D TMA boxes (codes, scales, biases; 64-bit
//    elements, box rows padded so that the lanes of one shared-memory read hit
//    distinct banks).  A CTA owns >= 16 rows; its last tile is moved up to end
//    on its last row, so it repeats a few rows just read (L2 hits, masked out
//    of the output) and never reads another CTA's rows.  The consumer warps
//    read the activations with plain loads (a copy through the copy engine
//    would queue behind the weight stages) and stage their digits in shared
//    memory.  Consumer warps (a divisor of the ring depth: one warp per slot)
//    take whole stages round-robin.  The chunks of one tile are summed in
//    chunk order through shared memory by the warp that handled the last chunk
//    (deterministic), then stored as bf16 (RNE).
//  * Sequence launches run up to four matmuls in one grid: the ring carries
//    their stages back to back, and a grid-wide barrier separates the end of
//    one matmul from the activation loads of the next.
//  * Every wait is bounded; a timeout sets a bit of g_qmv_tc_fault.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace aq {

__device__ uint32_t g_qmv_tc_fault = 0;

namespace qmm {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();  // driver entry point, resolved once (qmm.cu)
}

namespace tc {

#ifndef AQ_QMV_MAX_CONSUMERS
#define AQ_QMV_MAX_CONSUMERS 12
#endif
#ifndef AQ_QMV_INFLIGHT
#define AQ_QMV_INFLIGHT 10
#endif
#ifndef AQ_QMV_STAGE_TARGET
#define AQ_QMV_STAGE_TARGET (16 * 1024)
#endif
constexpr int kRows = 16;           // rows of W per tile (the MMA's M)
constexpr int kMaxConsumers = AQ_QMV_MAX_CONSUMERS;  // consumer warps per CTA at most
constexpr int kRedBufs = 4;         // tiles whose partial sums can be in flight
constexpr int kDualSmem = 112 * 1024;   // shared memory of a CTA that shares its SM with the next launch's
constexpr int kDualConsumers = 8;       // consumer warps of such a CTA
constexpr int kDualMinStages = 4;
constexpr int kUnitCodes = 1 << 20;     // codes of a row a work unit covers at most: a whole stage
#ifndef AQ_QMV_SMALL_UNIT
#define AQ_QMV_SMALL_UNIT 1024           // codes of a row per work unit where smaller units pay (unit_codes)
#endif
constexpr int kMaxStages = 16;
// Weight stages the producer keeps in flight (issued, not yet landed).  Enough
// to cover HBM latency at an SM's share of the bandwidth; more only lengthens
// the queue that every other load of the SM (activations, barrier traffic)
// waits behind.  Measured on B200 (decode step, 4-bit G64): 4 / 6 / 8 / 10 /
// 12 / 16 stages: 28.6 / 27.35 / 27.3 / 26.8 / 26.8 / 26.8 us (the long-K linear
// gains; the other shapes and the small-M curves do not move from 6 up).
constexpr int kInflight = AQ_QMV_INFLIGHT;
constexpr int kStageTarget = AQ_QMV_STAGE_TARGET;  // packed bytes of one stage we aim for (<= 1 KB per row)
constexpr int kAcc = 2;                  // independent accumulator chains per digit plane
constexpr int kStageItems = 2;           // activation staging items per thread per round          // weight stages issued before the previous kernel completes (overlap mode)
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds |v| < 2^22 to an integer

__host__ __device__ constexpr int pow2_tokens(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

// Packed words of one group row that one lane reads, and the first of them.
template <int BITS, int G>
struct LaneWords {
  static constexpr int count = BITS == 4 ? G / 32 : BITS == 8 ? G / 16 : (G >= 64 ? G / 64 : 1);
  AQ_DEVICE static int first(int t) { return (BITS == 2 && G == 32) ? (t >> 1) : t * count; }
};

// Activations one lane stages per group: a run of consecutive elements
// starting at start(t); element index(c, s, i, hh) of that run meets byte i of
// A register set s (s = 0: MMA k 4t..4t+3, s = 1: k 16+4t..16+4t+3) of the
// lane's K tile c (32 codes).  hh: the half of a shared word that a lane of a
// 2-bit, G = 32 pair owns (t & 1).
// FMT 1, 2 (mxfp4, nvfp4; 4-bit codes, 32-code spans): register set s holds
// codes 4s..4s+3 of the lane's word.  FMT 3 (mxfp8): staged slot s holds
// elements 4s..4s+3 of the lane's run as two fp16 pairs.
template <int BITS, int G, int FMT = 0>
struct LaneSpan {
  static constexpr int length = (BITS == 2 && G == 32) ? 16 : G / 4;
  AQ_DEVICE static int start(int t) { return (BITS == 2 && G == 32) ? 16 * (t >> 1) : t * (G / 4); }
  __host__ __device__ static constexpr int index(int c, int s, int i, int hh) {
    return FMT >= 1    ? 8 * c + 4 * s + i
           : BITS == 4 ? 8 * c + 2 * i + s
           : BITS == 8 ? 4 * (2 * c + s) + i
           : G >= 64   ? 16 * (c >> 1) + 2 * (c & 1) + s + 4 * i
                       : 2 * hh + s + 4 * i;
  }
};

template <int N>
AQ_DEVICE void lds_words(const uint8_t *p, uint32_t (&w)[N]) {
  if constexpr (N == 1) {
    w[0] = *reinterpret_cast<const uint32_t *>(p);
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4 *>(p)[i];
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
}

// The codes of K tile C of one row as bytes: a[0] = the 4 codes of register
// set 0, a[1] = set 1 (positions as in LaneSpan::index).
template <int BITS, int G, int C>
AQ_DEVICE void tile_codes(const uint32_t (&w)[LaneWords<BITS, G>::count], int t, uint32_t (&a)[2]) {
  if constexpr (BITS == 4) {
    a[0] = w[C] & 0x0F0F0F0Fu;
    a[1] = (w[C] >> 4) & 0x0F0F0F0Fu;
  } else if constexpr (BITS == 8) {
    a[0] = w[2 * C];
    a[1] = w[2 * C + 1];
  } else if constexpr (G == 32) {
    const uint32_t v = w[0] >> ((t & 1) * 4);
    a[0] = v & 0x03030303u;
    a[1] = (v >> 2) & 0x03030303u;
  } else {
    const uint32_t v = (C & 1) ? (w[C >> 1] >> 4) : w[C >> 1];
    a[0] = v & 0x03030303u;
    a[1] = (v >> 2) & 0x03030303u;
  }
}

// d += A(16x32 u8) * B(32x8), B unsigned (u8) or signed (s8) bytes; int32 accumulate.
AQ_DEVICE void mma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
AQ_DEVICE void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// prmt.b32 in its default mode: result byte n is byte (c >> 4n) & 7 of {b, a},
// or, when bit 4n+3 of c is set, that byte's sign bit replicated.
AQ_DEVICE uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight E2M1 codes of a word (nibbles: sign bit 3, magnitude bits 2..0) as their
// doubled magnitudes 2 * {0, 0.5, 1, 1.5, 2, 3, 4, 6} = 0..12 in unsigned bytes,
// split by sign: pos holds the positive codes (0 for the negative ones), neg the
// negative ones.  Register set s takes codes 4s..4s+3.  One prmt looks up four
// codes; a set sign bit replicates the table byte's clear sign bit, giving 0, so
// the lookup with the sign bits flipped keeps exactly the negative codes.
AQ_DEVICE void e2m1x2_split(uint32_t w, uint32_t (&pos)[2], uint32_t (&neg)[2]) {
  constexpr uint32_t kLo = 0x03020100u, kHi = 0x0C080604u;
  const uint32_t wn = w ^ 0x88888888u;
  pos[0] = prmt(kLo, kHi, w);
  neg[0] = prmt(kLo, kHi, wn);
  pos[1] = prmt(kLo, kHi, w >> 16);
  neg[1] = prmt(kLo, kHi, wn >> 16);
}

// d += A(16x16 f16) * B(16x8 f16), fp32 accumulate (mxfp8: E4M3 codes widened to fp16).
AQ_DEVICE void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two E4M3 codes (the low 16 bits of w: first code in the low byte) as fp16x2,
// first code in the low half (exact: E4M3 values are fp16 values).
AQ_DEVICE uint32_t e4m3x2_to_f16x2(uint32_t w) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// X of an E8M0 scale byte (s = 0: 2^-127, a subnormal; 255: NaN).
AQ_DEVICE float e8m0_full(uint32_t sb) {
  return sb == 0u ? __uint_as_float(0x00400000u) : (sb == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float(sb << 23));
}

// Half of an E4M3 scale byte's value (sign 0, exponent bits 6..3 with bias 7,
// mantissa bits 2..0; subnormals m * 2^-9; 0x7F is NaN).
AQ_DEVICE float e4m3_half(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (b == 0x7Fu) return __uint_as_float(0x7FC00000u);
  return e == 0u ? __uint_as_float(0x3A800000u) * static_cast<float>(m)   // m * 2^-10
                 : __uint_as_float(((e + 119u) << 23) | (m << 20));
}

// X / 2 of an E8M0 scale byte (X = 2^(s - 127); the MMA sees values doubled).
AQ_DEVICE float e8m0_half(uint32_t sb) {
  return sb >= 2u ? (sb == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float((sb - 1u) << 23))
                  : __uint_as_float(0x00200000u << sb);
}

// Bounded spin until *ctr >= target (shared-memory counter written by other
// warps of the CTA); false on timeout (fault bit set, abort raised) or abort.
AQ_DEVICE bool spin_until_at_least(int *ctr, int target, volatile int *abort_flag, long long limit) {
  volatile int *c = ctr;
  if (*c >= target) return true;
  const long long t0 = clock64();
  while (*c < target) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      atomicOr(&g_qmv_tc_fault, kFaultQmvWait);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// One matmul of a launch.  A sequence launch runs several, in order: the
// activations of matmul j are read only after every output of matmul j - 1 is
// complete (so y of one may be x of the next), while the weights of matmul j
// stream into the ring as soon as it has room.
struct Job {
  const __nv_bfloat16 *x;
  __nv_bfloat16 *y;
  int N, K, Gn;
  int Kc, nch;               // K chunk of a stage, chunks per row
  int fpu;                   // folds per work unit
  int parts;                 // units per 16-row tile (nch * nper): partial sums reduced per tile
  int pitch_w, pitch_s;      // bytes per row of codes / of scales (biases) in a stage
  int s_off, b_off;          // scales and biases inside a stage
  int tok_stride;            // staged activations: token m at xs_off + m * tok_stride
  int w_box_x, sb_box_x;     // TMA x coordinate step of one chunk (64-bit elements)
};
constexpr int kSeqMax = 4;   // matmuls of one sequence launch at most

template <int NJ>
struct JobMaps {
  CUtensorMap w[NJ], s[NJ], b[NJ];  // codes, scales, biases of each matmul
};

struct Args {
  Job job[kSeqMax];
  int njobs;
  unsigned *gbar;            // sequence launches: grid barrier (count, generation) between matmuls
  int M;
  int W, NS;                 // consumer warps, ring stages
  int nper;                  // work units per stage
  int red_bufs;              // tiles whose partials can be in flight at once
  long long wait_cycles;     // limit of every bounded wait, in SM clock cycles
  int stall;                 // nonzero: the consumers also wait on a barrier nothing completes (timeout test)
  int stage_bytes;
  int xs_off;
  int zero_off, zero_stride; // two zero blocks
  int tab_off, red_off, bar_off;
  // gather mode (cta_per_tok > 0): token t = blockIdx.x / cta_per_tok multiplies
  // its x row by expert experts[t] of E stacked [N, K] weights (rows e*N.. of
  // the [E*N, K] maps); each of its cta_per_tok CTAs owns a slice of the N rows
  const int32_t *experts;
  int E, cta_per_tok;
  const float *gscale;  // nvfp4: the tensor scale (device), applied to every output
};

// Grid-wide barrier of a sequence launch (every CTA of the grid is resident:
// one CTA per SM, at most one per SM fits).  gbar[0] counts arrivals, gbar[1]
// is the generation; the last arrival resets the count and advances the
// generation, so the pair is ready for the next barrier and the next launch.
// Bounded: false after `limit` cycles (fault bit set, abort raised).
AQ_DEVICE unsigned ld_acquire_gpu(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
AQ_DEVICE unsigned atom_add_acq_rel_gpu(unsigned *p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
AQ_DEVICE bool grid_barrier(unsigned *gbar, unsigned nblocks, volatile int *abort_flag, long long limit) {
  const unsigned g0 = ld_acquire_gpu(gbar + 1);
  // release: this CTA's outputs (ordered before by the CTA barrier) go with the arrival
  if (atom_add_acq_rel_gpu(gbar, 1u) == nblocks - 1) {
    atomicExch(gbar, 0u);
    atom_add_acq_rel_gpu(gbar + 1, 1u);
    return true;
  }
  const long long t0 = clock64();
  while (ld_acquire_gpu(gbar + 1) == g0) {
    if (*abort_flag || clock64() - t0 > limit) {
      atomicOr(&g_qmv_tc_fault, kFaultQmvWait);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

template <int BITS, int G, int MP, int FMT, int NJ = 1>
__global__ void __launch_bounds__(32 * (kMaxConsumers + 1), 1) qmv_tc_kernel(const __grid_constant__ Args a,
                                                                  const __grid_constant__ JobMaps<NJ> mp) {
  constexpr int GS = 8 / MP;                     // groups side by side in one accumulator
  constexpr int U = G / 32;                      // K tiles (16 bytes of activation digits per lane) per group
  constexpr int NWD = LaneWords<BITS, G>::count;
  constexpr int GBYTES = G * BITS / 8;           // packed bytes of one group row
  constexpr int SL = LaneSpan<BITS, G, FMT>::length;
  static_assert(FMT == 0 || FMT == 3 || (BITS == 4 && G == 32), "mxfp4 / nvfp4: 4-bit codes in 32-code spans");
  static_assert(FMT != 3 || (BITS == 8 && G == 32), "mxfp8: 8-bit codes, groups of 32");
  // nvfp4: a 32-code span holds two 16-weight groups, fed to two columns of one MMA
  static_assert(FMT != 2 || MP <= 4, "nvfp4 needs two group slots per token");
  // accumulator chains per digit plane: a group folded on its own has only
  // G/32 MMAs per plane, and summing chains would cost more than it hides
  constexpr int NACC = GS == 1 ? 1 : kAcc;
  // Affine codes (FMT 0): both digit planes go through one MMA, in adjacent
  // columns (column 2p + d: position p, digit d, both digits signed bytes), so
  // one MMA per K tile serves up to four tokens.  Position p is token p / GS1,
  // group slot p % GS1 of the fold.
  constexpr int TPM = MP >= 4 ? 4 : MP;   // tokens per MMA
  constexpr int NMMA = MP > 4 ? 2 : 1;    // MMAs per K tile (token halves)
  constexpr int GS1 = 4 / TPM;            // group slots per fold
  constexpr int NACC1 = GS1 == 1 ? 1 : GS1 == 4 ? 4 : kAcc;  // one token: four chains of two MMAs per fold
  using Span = LaneSpan<BITS, G, FMT>;

  extern __shared__ __align__(128) uint8_t smem[];
  // The tensor maps live in the launch's parameters, which a decode launch
  // finds cold in every cache: start fetching them before anything else (the
  // first copy would otherwise wait for the parameter read, then for the map).
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.w[0])) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.s[0])) : "memory");
    if constexpr (FMT == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.b[0])) : "memory");
  }
  // The other parameters are cold too, and the prologue reads them one after
  // another (ring depth, the matmul's fields, offsets), each read waiting for
  // its own miss.  One load per 64-byte line, issued side by side by threads
  // of the first consumer warp whose results nothing waits for, brings them in
  // together (measured: 0.3-0.6 us less per decode launch).
  {
    constexpr int kLines = static_cast<int>((sizeof(Args) + 63) / 64);
    static_assert(kLines <= 32, "one warp warms the parameter lines");
    if (threadIdx.x >= 32 && threadIdx.x < 32 + kLines) {
      const uint8_t *line = reinterpret_cast<const uint8_t *>(&a) + (threadIdx.x - 32) * 64;
      uint32_t unused;
      asm volatile("ld.b32 %0, [%1];" : "=r"(unused) : "l"(line) : "memory");
    }
  }
  uint8_t *ring = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + a.bar_off);
  uint64_t *empty = full + a.NS;
  uint64_t *stall_bar = empty + a.NS;  // no thread ever arrives on it (the timeout test waits on it)
  // chunk partials of a tile: red_ready[b] counts partials written into buffer
  // b, red_done[b] the tiles summed out of it (monotonic, so a waiter can never
  // mistake an older round for the one it needs)
  int *red_ready = reinterpret_cast<int *>(stall_bar + 2);  // (one barrier slot spare)
  int *red_done = red_ready + a.red_bufs;
  volatile int *abort_flag = red_done + a.red_bufs;
  int *issued_ctr = red_done + a.red_bufs + 1;  // stages the producer issued (read after an abort)
  uint8_t *xs = smem + a.xs_off;
  uint8_t *zero = smem + a.zero_off;
  float4 *tab = reinterpret_cast<float4 *>(smem + a.tab_off);  // [MP][Gn]: (sum x, 2^-e_lo, 2^-e_hi, 0)
  float *red = reinterpret_cast<float *>(smem + a.red_off);    // [red_bufs][parts][16][MP]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Job &J0 = a.job[0];
  // matmul jx's fields, by value: read from the parameters once per matmul (a
  // single-matmul launch indexes them at compile-time offsets)
  auto job_of = [&](int jx) -> Job { return a.job[NJ == 1 ? 0 : jx]; };
  int64_t gr0 = 0, gr1 = 0, wrow0 = 0;  // gather mode: rows [gr0, gr1) of this CTA; first row of its expert
  const __nv_bfloat16 *xg = J0.x;       // gather mode: this CTA's token row
  __nv_bfloat16 *yg0 = J0.y;
  if (a.cta_per_tok > 0) {
    const int tk = blockIdx.x / a.cta_per_tok, sub = blockIdx.x - tk * a.cta_per_tok;
    gr0 = static_cast<int64_t>(sub) * J0.N / a.cta_per_tok;
    gr1 = static_cast<int64_t>(sub + 1) * J0.N / a.cta_per_tok;
    xg = J0.x + static_cast<int64_t>(tk) * J0.K;
    yg0 = J0.y + static_cast<int64_t>(tk) * J0.N;
    const int e = __ldg(a.experts + tk);
    if (e < 0 || e >= a.E) {  // bad expert id: zero rows and a fault bit, before anything is issued
      for (int64_t r = gr0 + threadIdx.x; r < gr1; r += blockDim.x) yg0[r] = __float2bfloat16_rn(0.0f);
      if (threadIdx.x == 0 && sub == 0) atomicOr(&g_qmv_tc_fault, kFaultBadIndex);
      return;
    }
    wrow0 = static_cast<int64_t>(e) * J0.N;
  }
  // rows [r0, r1) of this CTA in matmul jx, and its stages (tiles x chunks)
  auto cta_rows = [&](int jx, int64_t &r0, int64_t &r1) {
    if (a.cta_per_tok > 0) {
      r0 = gr0;
      r1 = gr1;
    } else {
      const uint32_t n = static_cast<uint32_t>(job_of(jx).N);
      if (n <= 0xFFFFFFFFu / gridDim.x) {  // 32-bit division (the 64-bit one is a long software routine)
        r0 = (blockIdx.x * n) / gridDim.x;
        r1 = ((blockIdx.x + 1) * n) / gridDim.x;
      } else {
        r0 = static_cast<int64_t>(blockIdx.x) * n / gridDim.x;
        r1 = static_cast<int64_t>(blockIdx.x + 1) * n / gridDim.x;
      }
    }
  };
  auto job_stages = [&](int jx) {
    int64_t r0, r1;
    cta_rows(jx, r0, r1);
    return static_cast<int>(static_cast<uint32_t>(r1 - r0 + kRows - 1) / kRows) * job_of(jx).nch;
  };
  const long long wlim = a.wait_cycles;

  // One stage: rows of codes, scales and biases of (tile, chunk); whole producer warp.
  // First W row of tile T.  A CTA owns >= 16 rows, so its last tile is moved
  // up to end at r1: its first rows repeat rows of the tile before (read again
  // from L2, not stored twice) and every stage is three whole TMA boxes.
  auto tile_base = [&](int64_t r0, int64_t r1, int T) { return min(r0 + static_cast<int64_t>(T) * kRows, r1 - kRows); };
  // One stage: 16 rows of codes, scales and biases of (tile, chunk) of matmul
  // jx, into ring slot gst % NS (gst counts the stages of all matmuls); one lane.
  auto issue = [&](int jx, const Job &Jb, int64_t r0, int64_t r1, int st, int gst) {
    const int s = gst % a.NS;
    const int T = st / Jb.nch, ch = st - T * Jb.nch;
    const int rb = static_cast<int>(wrow0 + tile_base(r0, r1, T));
    uint8_t *dst = ring + static_cast<size_t>(s) * a.stage_bytes;
    mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kRows * (Jb.pitch_w + (FMT == 0 ? 2 : 1) * Jb.pitch_s)));
    tma_load_2d(dst, &mp.w[NJ == 1 ? 0 : jx], &full[s], ch * Jb.w_box_x, rb);
    tma_load_2d(dst + Jb.s_off, &mp.s[NJ == 1 ? 0 : jx], &full[s], ch * Jb.sb_box_x, rb);
    if constexpr (FMT == 0) tma_load_2d(dst + Jb.b_off, &mp.b[NJ == 1 ? 0 : jx], &full[s], ch * Jb.sb_box_x, rb);
  };

  if (tid == 0) {
    for (int s = 0; s < a.NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], a.nper);  // every unit (fold) of a stage releases it once
    }
    for (int b = 0; b < a.red_bufs; ++b) red_ready[b] = red_done[b] = 0;
    mbar_init(stall_bar, 1);
    *abort_flag = 0;
    *issued_ctr = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // A kernel launched after this one as a programmatic dependent may start its
  // prologue now; it waits for this grid before reading anything it writes.
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Every stage of every matmul in order, each as soon as its ring slot is
    // free.  The weights are not written by a kernel this one may overlap (the
    // caller's promise for programmatic dependent launches), so the producer
    // does not wait for the kernel before; the activations are loaded by the
    // consumers, outside the copy engine, so they never queue behind weights.
    if (lane == 0) {
      int gst = 0;
      bool ok = true;
      for (int jx = 0; jx < a.njobs && ok; ++jx) {
        const Job jb = job_of(jx);
        int64_t q0, q1;
        cta_rows(jx, q0, q1);
        const int nstj = job_stages(jx);
        for (int st = 0; st < nstj; ++st, ++gst) {
          const int s = gst % a.NS;
          if (gst >= a.NS &&
              !mbar_wait(&empty[s], ((gst / a.NS) - 1) & 1, abort_flag, &g_qmv_tc_fault, kFaultQmvWait, wlim)) {
            ok = false;
            break;
          }
          // the stage kInflight back has landed (its slot is issued again only
          // NS > kInflight stages later, so the phase waited for is current)
          const int back = gst - kInflight;
          if (back >= 0 && kInflight < a.NS &&
              !mbar_wait(&full[back % a.NS], (back / a.NS) & 1, abort_flag, &g_qmv_tc_fault, kFaultQmvWait, wlim)) {
            ok = false;
            break;
          }
          issue(jx, jb, q0, q1, st, gst);
        }
      }
      *issued_ctr = gst;
    }
    __syncwarp();
  } else {

  // ---- consumers stage the activations: item = (token, group, lane t).  The
  // raw bf16 values come straight from global memory (plain loads: the
  // activations of a later matmul were written by other CTAs of this launch,
  // made visible by the grid barrier), the digits go to shared memory.
  const int ctid = tid - 32, cthreads = a.W * 32;
  auto stage_acts = [&](int jx) {
    const Job Jb = job_of(jx);
    // x of the first matmul may be the output of the kernel this one overlaps
    if (jx == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    const __nv_bfloat16 *xsrc = (a.cta_per_tok > 0) ? xg : Jb.x;
    const int items = a.M * Jb.Gn * 4;  // a multiple of 4, so the 4 items of a group share one quad of lanes
    // Each thread takes kStageItems items per round, processed side by side:
    // the rounds are latency-bound chains (load, reduce across the quad, store).
    constexpr int NI = kStageItems;
    for (int i0 = 0; i0 < items; i0 += NI * cthreads) {
      int tq[NI], mq[NI], gq[NI];
      bool act[NI];
      uint32_t raw[NI][SL / 2];
      static_for<0, NI>([&](auto J) {
        constexpr int j = J.value;
        const int i = i0 + j * cthreads + ctid;
        act[j] = i < items;
        const int ii = act[j] ? i : 0;
        tq[j] = ii & 3;
        const int mg = ii >> 2;
        mq[j] = mg / Jb.Gn;
        gq[j] = mg - mq[j] * Jb.Gn;
        const uint4 *src = reinterpret_cast<const uint4 *>(xsrc + static_cast<int64_t>(mq[j]) * Jb.K + gq[j] * G +
                                                           Span::start(tq[j]));
#pragma unroll
        for (int v = 0; v < SL / 8; ++v) {
          const uint4 q = act[j] ? src[v] : make_uint4(0u, 0u, 0u, 0u);
          raw[j][4 * v] = q.x;
          raw[j][4 * v + 1] = q.y;
          raw[j][4 * v + 2] = q.z;
          raw[j][4 * v + 3] = q.w;
        }
      });
      float v8[NI][U][8];  // [item][tile][4 * set + byte]
      float amax[NI], sx[NI];
      static_for<0, NI>([&](auto J) {
        constexpr int j = J.value;
        amax[j] = 0.0f;
        sx[j] = 0.0f;
        static_for<0, U>([&](auto C) {
          static_for<0, 8>([&](auto S) {
            constexpr int c = C.value, st = S.value >> 2, i = S.value & 3;
            constexpr int e0 = Span::index(c, st, i, 0), e1 = Span::index(c, st, i, 1);
            const uint32_t r0v = raw[j][e0 >> 1] >> ((e0 & 1) * 16), r1v = raw[j][e1 >> 1] >> ((e1 & 1) * 16);
            const uint32_t bits16 = (e0 == e1 || !(tq[j] & 1)) ? r0v : r1v;
            const float v = bf16_bits_to_float(bits16 & 0xFFFFu);
            v8[j][c][S.value] = v;
            amax[j] = fmaxf(amax[j], fabsf(v));
            sx[j] += v;
          });
        });
      });
      __syncwarp();  // every lane of the warp has read its raw values
      static_for<0, NI>([&](auto J) {
        constexpr int j = J.value;
        amax[j] = fmaxf(amax[j], __shfl_xor_sync(0xffffffffu, amax[j], 1));
        sx[j] += __shfl_xor_sync(0xffffffffu, sx[j], 1);
      });
      static_for<0, NI>([&](auto J) {
        constexpr int j = J.value;
        amax[j] = fmaxf(amax[j], __shfl_xor_sync(0xffffffffu, amax[j], 2));
        sx[j] += __shfl_xor_sync(0xffffffffu, sx[j], 2);
      });
      static_for<0, NI>([&](auto J) {
        constexpr int j = J.value;
        // power of two 2^e with max|x| * 2^e in [2^13, 2^14) (e clamped to normal fp32 powers)
        int e = 0;
        if (amax[j] > 0.0f) {
          const int be = static_cast<int>((__float_as_uint(amax[j]) >> 23) & 0xFFu);
          e = min(max(13 - (be == 0 ? -127 : be - 127), -126), 126);
        }
        // 2^-e as 2^-e_lo * 2^-e_hi: the fold applies one half to the integer dot
        // product and the other to the scale, so neither product leaves fp32 range
        const int e_hi = e >> 1, e_lo = e - e_hi;
        const float inv_lo = __uint_as_float(static_cast<uint32_t>(127 - e_lo) << 23);
        const float inv_hi = __uint_as_float(static_cast<uint32_t>(127 - e_hi) << 23);
        const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
        uint8_t *dst = xs + mq[j] * Jb.tok_stride + (gq[j] * U) * 64 + tq[j] * 16;
        static_for<0, U>([&](auto C) {
          constexpr int c = C.value;
          if constexpr (FMT == 3) {  // fp16 pairs (elements 2i, 2i+1) of x * 2^e: exact in fp16's normal range
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const __half2 p = __floats2half2_rn(v8[j][c][2 * i] * sc, v8[j][c][2 * i + 1] * sc);
              h[i] = *reinterpret_cast<const uint32_t *>(&p);
            }
            if (act[j]) *reinterpret_cast<uint4 *>(dst + c * 64) = make_uint4(h[0], h[1], h[2], h[3]);
            return;
          }
          uint32_t lo[2], hi[2];
          static_for<0, 2>([&](auto S) {
            // x_int = rint(v * 2^e) lands in the low 22 bits of v * 2^e + 1.5 * 2^23
            // (two's complement).  Signed digits x_int = 256 * hi + lo with lo in
            // [-128, 127] and hi in [-64, 64]: lo is byte 0 of x_int, hi is
            // byte 1 of x_int + 128 (an integer add on the bit pattern).
            uint32_t f[4], f2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              f[i] = __float_as_uint(fmaf(v8[j][c][4 * S.value + i], sc, kRoundMagic));
              f2[i] = f[i] + 128u;
            }
            const uint32_t t01 = __byte_perm(f[0], f[1], 0x40), t23 = __byte_perm(f[2], f[3], 0x40);
            const uint32_t u01 = __byte_perm(f2[0], f2[1], 0x51), u23 = __byte_perm(f2[2], f2[3], 0x51);
            lo[S.value] = __byte_perm(t01, t23, 0x5410);
            hi[S.value] = __byte_perm(u01, u23, 0x5410);
          });
          if (act[j]) *reinterpret_cast<uint4 *>(dst + c * 64) = make_uint4(lo[0], lo[1], hi[0], hi[1]);
        });
        if (act[j] && tq[j] == 0) tab[mq[j] * Jb.Gn + gq[j]] = make_float4(sx[j], inv_lo, inv_hi, 0.0f);
      });
    }
    // zero blocks, and the table rows of padding tokens
    const int zbytes = a.zero_stride + U * 64;
    for (int i = ctid; i < zbytes / 16; i += cthreads) reinterpret_cast<uint4 *>(zero)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = a.M * Jb.Gn + ctid; i < MP * Jb.Gn; i += cthreads) tab[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // all consumer warps (not the producer) meet here: the staged activations are complete
    asm volatile("bar.sync 1, %0;" ::"r"(cthreads) : "memory");
  };
  stage_acts(0);
  // timeout test: a wait on a barrier that nothing completes runs out, raises
  // the abort flag and sets the fault bit; every other wait then gives up
  if (a.stall) mbar_wait(stall_bar, 0, abort_flag, &g_qmv_tc_fault, kFaultQmvWait, wlim);

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int g = lane >> 2, t = lane & 3;
  const int my_m = g / GS, my_j = g % GS;          // this lane's B column: token, group slot
  const bool my_real = my_m < a.M;
  const uint8_t *zero_lane = zero + (GS == 1 ? 0 : (my_m & 1)) * a.zero_stride + t * 16;
  const int lw0 = LaneWords<BITS, G>::first(t) * 4;
  constexpr int SPANS = FMT == 0 ? GS1 : FMT == 2 ? GS / 2 : GS;  // 32-code spans (MMA K steps) per fold
  const float gs = FMT == 2 ? __ldg(a.gscale) : 1.0f;
  // FMT 0: B column g = 2p + d of this lane (token, slot and digit plane it
  // feeds) and the accumulator columns 2t, 2t+1 it receives (position t)
  const int b_slot = (g >> 1) % GS1;
  int b_tok[NMMA];
#pragma unroll
  for (int h = 0; h < NMMA; ++h) b_tok[h] = h * 4 + (g >> 1) / GS1;
  const uint8_t *zb_lane = zero + t * 16 + (g & 1) * 8;
  const int c_slot = t % GS1;

  // Work units: unit u is fold p of stage st (u = st * nper + p), dealt to the
  // consumer warps round-robin, so a stage is shared by several warps and the
  // last stages of a launch spread over all of them.  W divides NS * nper, so
  // the units a warp meets in one ring slot are consecutive phases of it.
  // Units are numbered across the matmuls of a launch (their stages follow one
  // another in the ring), so warp cw takes global units cw, cw + W, ...
  int gbase = 0;  // stages of the matmuls before this one
  bool run = true;
  // Every consumer warp walks every matmul, also after a failed wait (then
  // without taking units), so that all of them meet at the named barriers.
  for (int jx = 0; jx < a.njobs; ++jx) {
  const Job Jb = job_of(jx);
  if (jx > 0) {
    // Every unit of matmul jx - 1 in this CTA is done (its outputs stored);
    // once every CTA is that far, the activations of matmul jx may be read.
    asm volatile("bar.sync 1, %0;" ::"r"(cthreads) : "memory");
    if (ctid == 0) {
      for (int b = 0; b < a.red_bufs; ++b) red_ready[b] = red_done[b] = 0;  // tile numbers restart
      grid_barrier(a.gbar, gridDim.x, abort_flag, wlim);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(cthreads) : "memory");  // ... and this CTA knows it
    __threadfence();
    stage_acts(jx);
    if (*abort_flag) run = false;
  }
  int64_t r0, r1;
  cta_rows(jx, r0, r1);
  const int nst = static_cast<int>(static_cast<uint32_t>(r1 - r0 + kRows - 1) / kRows) * Jb.nch;
  const int gpc = Jb.Kc / G;  // groups per chunk
  __nv_bfloat16 *yg = a.cta_per_tok > 0 ? yg0 : Jb.y;
  const uint8_t *xs_lane = xs + (my_real ? my_m : 0) * Jb.tok_stride + t * 16;
  const uint8_t *b_lane[NMMA];
#pragma unroll
  for (int h = 0; h < NMMA; ++h) b_lane[h] = xs + (b_tok[h] < a.M ? b_tok[h] : 0) * Jb.tok_stride + t * 16 + (g & 1) * 8;
  const int nunits = nst * a.nper;
  const int ubase = gbase * a.nper;
  for (int u = ((cw - ubase) % a.W + a.W) % a.W; run && u < nunits; u += a.W) {
    const int st = u / a.nper, p = u - st * a.nper;
    const int gst = gbase + st;
    const int s = gst % a.NS;
    if (!mbar_wait(&full[s], (gst / a.NS) & 1, abort_flag, &g_qmv_tc_fault, kFaultQmvWait, wlim)) {
      run = false;
      break;
    }
    const int T = st / Jb.nch, ch = st - T * Jb.nch;
    const int64_t rb = tile_base(r0, r1, T);
    const int v0 = static_cast<int>(r0 + static_cast<int64_t>(T) * kRows - rb);  // rows [v0, 16) are new
    auto row_ok = [&](int r) { return r >= v0 && rb + r < r1; };
    const uint8_t *stg = ring + static_cast<size_t>(s) * a.stage_bytes;
    const uint8_t *wr0 = stg + g * Jb.pitch_w + lw0;
    const uint8_t *wr1 = wr0 + 8 * Jb.pitch_w;
    const uint8_t *sr0 = stg + Jb.s_off + g * Jb.pitch_s, *sr1 = sr0 + 8 * Jb.pitch_s;
    const uint8_t *br0 = stg + Jb.b_off + g * Jb.pitch_s, *br1 = br0 + 8 * Jb.pitch_s;
    const int gch0 = ch * gpc;
    // Per (row, token) partials of this unit, held by some lanes: value q is
    // (row vrow[q], token vtok[q]) of the tile.
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int vrow[4] = {0, 0, 0, 0}, vtok[4] = {0, 0, 0, 0};
    int nv = 0;
    bool holder = false;
    if constexpr (FMT == 0) {
      float2 acc1[NMMA];  // rows (g, g+8) of token h * 4 + t / GS1
#pragma unroll
      for (int h = 0; h < NMMA; ++h) acc1[h] = make_float2(0.0f, 0.0f);
      for (int pf = p * Jb.fpu; pf < (p + 1) * Jb.fpu; ++pf) {  // the unit's folds
        int dd[NMMA][NACC1][4];  // (lo, hi) digit sums of rows g and g+8 at position t
#pragma unroll
        for (int h = 0; h < NMMA; ++h)
#pragma unroll
          for (int i = 0; i < NACC1; ++i) dd[h][i][0] = dd[h][i][1] = dd[h][i][2] = dd[h][i][3] = 0;
        static_for<0, SPANS>([&](auto J) {
          constexpr int j = J.value;
          const int gi = pf * SPANS + j;
          uint32_t w0[NWD], w1[NWD];
          lds_words<NWD>(wr0 + gi * GBYTES, w0);
          lds_words<NWD>(wr1 + gi * GBYTES, w1);
          static_for<0, U>([&](auto C) {
            constexpr int c = C.value;
            constexpr int k = (j * U + c) % NACC1;
            uint32_t q0[2], q1[2];
            tile_codes<BITS, G, c>(w0, t, q0);
            tile_codes<BITS, G, c>(w1, t, q1);
            static_for<0, NMMA>([&](auto H) {
              constexpr int h = H.value;
              const bool live = b_slot == j && b_tok[h] < a.M;
              const uint8_t *bp = live ? b_lane[h] + (gch0 + gi) * (U * 64) + c * 64 : zb_lane + c * 64;
              const uint2 bv = *reinterpret_cast<const uint2 *>(bp);
              mma_u8s8(dd[h][k], q0[0], q1[0], q0[1], q1[1], bv.x, bv.y);
            });
          });
        });
        // fold: y += (s * 2^-e_hi) * (D * 2^-e_lo) + b * sum x, rows g and g+8 side by side
        const int gl = pf * SPANS + c_slot;
        const float2 sv = make_float2(__half2float(*reinterpret_cast<const __half *>(sr0 + gl * 2)),
                                      __half2float(*reinterpret_cast<const __half *>(sr1 + gl * 2)));
        const float2 bv2 = make_float2(__half2float(*reinterpret_cast<const __half *>(br0 + gl * 2)),
                                       __half2float(*reinterpret_cast<const __half *>(br1 + gl * 2)));
#pragma unroll
        for (int h = 0; h < NMMA; ++h) {
          int lo0 = dd[h][0][0], hi0 = dd[h][0][1], lo1 = dd[h][0][2], hi1 = dd[h][0][3];
#pragma unroll
          for (int i = 1; i < NACC1; ++i) {
            lo0 += dd[h][i][0];
            hi0 += dd[h][i][1];
            lo1 += dd[h][i][2];
            hi1 += dd[h][i][3];
          }
          const float2 D = make_float2(static_cast<float>(lo0 + 256 * hi0), static_cast<float>(lo1 + 256 * hi1));
          const float4 T4 = tab[(h * 4 + t / GS1) * Jb.Gn + gch0 + gl];
          acc1[h] = ffma2(__fmul2_rn(sv, make_float2(T4.z, T4.z)), __fmul2_rn(D, make_float2(T4.y, T4.y)),
                          ffma2(bv2, make_float2(T4.x, T4.x), acc1[h]));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // the lanes of one token (t / GS1 equal) sum their group slots
#pragma unroll
      for (int h = 0; h < NMMA; ++h) {
        float e0 = acc1[h].x, e1 = acc1[h].y;
        if constexpr (GS1 >= 2) {
          e0 += __shfl_xor_sync(0xffffffffu, e0, 1);
          e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
        }
        if constexpr (GS1 >= 4) {
          e0 += __shfl_xor_sync(0xffffffffu, e0, 2);
          e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
        }
        v[2 * h] = e0;
        v[2 * h + 1] = e1;
        vrow[2 * h] = g;
        vrow[2 * h + 1] = g + 8;
        vtok[2 * h] = vtok[2 * h + 1] = h * 4 + t / GS1;
      }
      nv = 2 * NMMA;
      holder = c_slot == 0;
    } else {
      float2 accA = make_float2(0.0f, 0.0f), accB = make_float2(0.0f, 0.0f);  // rows g, g+8 x columns 2t, 2t+1

      for (int pf = p * Jb.fpu; pf < (p + 1) * Jb.fpu; ++pf) {  // the unit's folds
        int dl[NACC][4], dh[NACC][4];  // sum q * lo, sum q * hi
        // mxfp4: the same sums over the negative codes' magnitudes, subtracted below
        int nl[FMT >= 1 ? NACC : 1][4], nh[FMT >= 1 ? NACC : 1][4];
        float fa[FMT == 3 ? NACC : 1][4];  // mxfp8: fp32 accumulators of the f16 MMAs
  #pragma unroll
        for (int i = 0; i < NACC; ++i) dl[i][0] = dl[i][1] = dl[i][2] = dl[i][3] = dh[i][0] = dh[i][1] = dh[i][2] = dh[i][3] = 0;
        if constexpr (FMT == 1 || FMT == 2) {
  #pragma unroll
          for (int i = 0; i < NACC; ++i) nl[i][0] = nl[i][1] = nl[i][2] = nl[i][3] = nh[i][0] = nh[i][1] = nh[i][2] = nh[i][3] = 0;
        }
        if constexpr (FMT == 3) {
  #pragma unroll
          for (int i = 0; i < NACC; ++i) fa[i][0] = fa[i][1] = fa[i][2] = fa[i][3] = 0.0f;
        }
        static_for<0, SPANS>([&](auto J) {
          constexpr int j = J.value;
          const int gi = pf * SPANS + j;
          uint32_t w0[NWD], w1[NWD];
          lds_words<NWD>(wr0 + gi * GBYTES, w0);
          lds_words<NWD>(wr1 + gi * GBYTES, w1);
          // nvfp4: the span's first 16 codes (lanes t = 0, 1) go to slot 2j, the
          // other 16 (t = 2, 3) to slot 2j + 1
          const bool live = my_real && (FMT == 2 ? my_j == 2 * j + (t >> 1) : my_j == j);
          const uint8_t *bp = live ? xs_lane + (gch0 + gi) * (U * 64) : zero_lane;
          static_for<0, U>([&](auto C) {
            constexpr int c = C.value;
            const uint4 bv = *reinterpret_cast<const uint4 *>(bp + c * 64);  // lo set 0, lo set 1, hi set 0, hi set 1
            uint32_t q0[2], q1[2];
            constexpr int k = (j * U + c) % NACC;
            if constexpr (FMT == 3) {
              // two k16 MMAs: codes 0..3 of the lane's run (words w[0]), then 4..7 (w[1])
              mma_f16(fa[k], e4m3x2_to_f16x2(w0[0]), e4m3x2_to_f16x2(w1[0]), e4m3x2_to_f16x2(w0[0] >> 16),
                      e4m3x2_to_f16x2(w1[0] >> 16), bv.x, bv.y);
              mma_f16(fa[(k + 1) % NACC], e4m3x2_to_f16x2(w0[1]), e4m3x2_to_f16x2(w1[1]), e4m3x2_to_f16x2(w0[1] >> 16),
                      e4m3x2_to_f16x2(w1[1] >> 16), bv.z, bv.w);
            } else if constexpr (FMT >= 1) {
              uint32_t n0[2], n1[2];
              e2m1x2_split(w0[0], q0, n0);
              e2m1x2_split(w1[0], q1, n1);
              mma_u8s8(dl[k], q0[0], q1[0], q0[1], q1[1], bv.x, bv.y);
              mma_u8s8(dh[k], q0[0], q1[0], q0[1], q1[1], bv.z, bv.w);
              mma_u8s8(nl[k], n0[0], n1[0], n0[1], n1[1], bv.x, bv.y);
              mma_u8s8(nh[k], n0[0], n1[0], n0[1], n1[1], bv.z, bv.w);
            }
          });
        });
        float D[4];  // sum_k q_k x_int_k of the lane's 4 (row, column) cells, exact in int32
  #pragma unroll
        for (int i = 0; i < 4; ++i) {
          int lo = dl[0][i], hi = dh[0][i];
  #pragma unroll
          for (int c = 1; c < NACC; ++c) {
            lo += dl[c][i];
            hi += dh[c][i];
          }
          if constexpr (FMT == 1 || FMT == 2) {
  #pragma unroll
            for (int c = 0; c < NACC; ++c) {
              lo -= nl[c][i];
              hi -= nh[c][i];
            }
          }
          if constexpr (FMT == 3) {  // fp32 sums of the f16 products
            float f = fa[0][i];
  #pragma unroll
            for (int c = 1; c < NACC; ++c) f += fa[c][i];
            D[i] = f;
          } else {
            D[i] = static_cast<float>(hi * 256 + lo);
          }
        }
        // fold: D[0] = (row g, col 2t), D[1] = (row g, col 2t+1), D[2], D[3] = rows g+8.
        // The two columns of a row go through packed fp32x2 operations.
        float2 s0, s1, b0, b1;  // scale and bias of (row g | g+8) for columns 2t, 2t+1
        float4 T0, T1;          // (sum x, 2^-e_lo, 2^-e_hi, 0) of columns 2t, 2t+1
        if constexpr (GS >= 2) {
          const int gl = pf * GS + (2 * t) % GS;  // group (in the chunk) of column 2t; 2t+1 is the next one
          const int mt = (2 * t) / GS;
          if constexpr (FMT == 2) {  // two E4M3 bytes per row (16-groups gl, gl + 1, one span); no bias
            const uint32_t e0 = *reinterpret_cast<const uint16_t *>(sr0 + gl);
            const uint32_t e1 = *reinterpret_cast<const uint16_t *>(sr1 + gl);
            s0 = make_float2(e4m3_half(e0 & 0xFFu), e4m3_half(e0 >> 8));
            s1 = make_float2(e4m3_half(e1 & 0xFFu), e4m3_half(e1 >> 8));
            b0 = b1 = make_float2(0.0f, 0.0f);
          } else if constexpr (FMT == 3) {  // two E8M0 bytes per row (groups gl, gl + 1): X; no bias
            const uint32_t e0 = *reinterpret_cast<const uint16_t *>(sr0 + gl);
            const uint32_t e1 = *reinterpret_cast<const uint16_t *>(sr1 + gl);
            s0 = make_float2(e8m0_full(e0 & 0xFFu), e8m0_full(e0 >> 8));
            s1 = make_float2(e8m0_full(e1 & 0xFFu), e8m0_full(e1 >> 8));
            b0 = b1 = make_float2(0.0f, 0.0f);
          } else if constexpr (FMT == 1) {  // two E8M0 bytes per row (groups gl, gl + 1); no bias
            const uint32_t e0 = *reinterpret_cast<const uint16_t *>(sr0 + gl);
            const uint32_t e1 = *reinterpret_cast<const uint16_t *>(sr1 + gl);
            s0 = make_float2(e8m0_half(e0 & 0xFFu), e8m0_half(e0 >> 8));
            s1 = make_float2(e8m0_half(e1 & 0xFFu), e8m0_half(e1 >> 8));
            b0 = b1 = make_float2(0.0f, 0.0f);
          } else {
            s0 = __half22float2(*reinterpret_cast<const __half2 *>(sr0 + gl * 2));
            s1 = __half22float2(*reinterpret_cast<const __half2 *>(sr1 + gl * 2));
            b0 = __half22float2(*reinterpret_cast<const __half2 *>(br0 + gl * 2));
            b1 = __half22float2(*reinterpret_cast<const __half2 *>(br1 + gl * 2));
          }
          if constexpr (FMT == 2) {  // both columns lie in span gl / 2 of the chunk
            T0 = T1 = tab[mt * Jb.Gn + gch0 + gl / 2];
          } else {
            T0 = tab[mt * Jb.Gn + gch0 + gl];
            T1 = tab[mt * Jb.Gn + gch0 + gl + 1];
          }
        } else {
          const int gl = pf;  // one group; columns 2t, 2t+1 are tokens 2t, 2t+1
          float sv0, sv1, bv0 = 0.0f, bv1 = 0.0f;
          if constexpr (FMT == 1) {
            sv0 = e8m0_half(sr0[gl]);
            sv1 = e8m0_half(sr1[gl]);
          } else if constexpr (FMT == 3) {
            sv0 = e8m0_full(sr0[gl]);
            sv1 = e8m0_full(sr1[gl]);
          } else {
            sv0 = __half2float(*reinterpret_cast<const __half *>(sr0 + gl * 2));
            sv1 = __half2float(*reinterpret_cast<const __half *>(sr1 + gl * 2));
            bv0 = __half2float(*reinterpret_cast<const __half *>(br0 + gl * 2));
            bv1 = __half2float(*reinterpret_cast<const __half *>(br1 + gl * 2));
          }
          s0 = make_float2(sv0, sv0);
          s1 = make_float2(sv1, sv1);
          b0 = make_float2(bv0, bv0);
          b1 = make_float2(bv1, bv1);
          T0 = tab[(2 * t) * Jb.Gn + gch0 + gl];
          T1 = tab[(2 * t + 1) * Jb.Gn + gch0 + gl];
        }
        const float2 tx = make_float2(T0.x, T1.x), ty = make_float2(T0.y, T1.y), tz = make_float2(T0.z, T1.z);
        // y += (s * 2^-e_hi) * (D * 2^-e_lo) + b * sum x   (block-scaled modes: no bias)
        if constexpr (FMT >= 1) {
          accA = ffma2(__fmul2_rn(s0, tz), __fmul2_rn(make_float2(D[0], D[1]), ty), accA);
          accB = ffma2(__fmul2_rn(s1, tz), __fmul2_rn(make_float2(D[2], D[3]), ty), accB);
        } else {
          accA = ffma2(__fmul2_rn(s0, tz), __fmul2_rn(make_float2(D[0], D[1]), ty), ffma2(b0, tx, accA));
          accB = ffma2(__fmul2_rn(s1, tz), __fmul2_rn(make_float2(D[2], D[3]), ty), ffma2(b1, tx, accB));
        }
      }
      const float acc[4] = {accA.x, accA.y, accB.x, accB.y};
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // Per (row, token) partials of this chunk: GS >= 2 sums the lane's two
      // columns (same token) and then the lanes sharing the token.
      if constexpr (GS >= 2) {
        v[0] = acc[0] + acc[1];
        v[1] = acc[2] + acc[3];
        if constexpr (GS >= 4) {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
          v[1] += __shfl_xor_sync(0xffffffffu, v[1], 1);
        }
        if constexpr (GS >= 8) {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
          v[1] += __shfl_xor_sync(0xffffffffu, v[1], 2);
        }
      } else {
        v[0] = acc[0];
        v[1] = acc[1];
        v[2] = acc[2];
        v[3] = acc[3];
      }
      // holder lanes: GS >= 2 -> lanes with t % (GS/2) == 0 hold (rows g, g+8; token 2t/GS)
      //               GS == 1 -> every lane holds (rows g, g+8; tokens 2t, 2t+1)
      holder = (GS == 1) || (t % (GS / 2 > 0 ? GS / 2 : 1) == 0);
      if constexpr (GS >= 2) {
        nv = 2;
        vrow[0] = g;
        vrow[1] = g + 8;
        vtok[0] = vtok[1] = (2 * t) / GS;
      } else {
        nv = 4;
  #pragma unroll
        for (int q = 0; q < 4; ++q) {
          vrow[q] = g + 8 * (q >> 1);
          vtok[q] = 2 * t + (q & 1);
        }
      }
    }
    auto put = [&](float *dstv, bool direct) {
      if (!holder) return;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q >= nv) break;
        if (direct) {
          if (vtok[q] < a.M && row_ok(vrow[q]))
            yg[static_cast<int64_t>(vtok[q]) * Jb.N + rb + vrow[q]] = __float2bfloat16_rn(FMT == 2 ? v[q] * gs : v[q]);
        } else {
          dstv[vrow[q] * MP + vtok[q]] = v[q];
        }
      }
    };
    if (Jb.parts == 1) {
      put(nullptr, true);
      continue;
    }
    const int b = T % a.red_bufs;
    const int rnd = T / a.red_bufs;
    // buffer b is free once the rnd earlier tiles that used it have been summed
    if (!spin_until_at_least(&red_done[b], rnd, abort_flag, wlim)) {
      run = false;
      break;
    }
    float *rbuf = red + static_cast<size_t>(b) * Jb.parts * kRows * MP;
    put(rbuf + static_cast<size_t>(ch * a.nper + p) * kRows * MP, false);
    __syncwarp();
    // The warp whose partial completes the tile sums all of them, in part
    // order (so the result does not depend on which warp finished last).
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&red_ready[b], 1) == (rnd + 1) * Jb.parts - 1;
      __threadfence_block();
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) continue;
    for (int idx = lane; idx < kRows * MP; idx += 32) {
      const int row = idx / MP, tok = idx - row * MP;
      float sum = 0.0f;
      for (int c2 = 0; c2 < Jb.parts; ++c2) sum += rbuf[(static_cast<size_t>(c2) * kRows + row) * MP + tok];
      if (tok < a.M && row_ok(row))
        yg[static_cast<int64_t>(tok) * Jb.N + rb + row] = __float2bfloat16_rn(FMT == 2 ? sum * gs : sum);
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      atomicAdd(&red_done[b], 1);
    }
  }
  gbase += nst;
  }  // matmuls
  }  // consumers

  // After an abort, copies that were issued but never consumed may still be
  // landing in this CTA's shared memory: wait for them (bounded) before the
  // CTA exits.  In a normal run every issued stage was awaited by a consumer.
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    const int issued = *issued_ctr;
    for (int j = max(0, issued - a.NS); j < issued; ++j) mbar_drain(&full[j % a.NS], (j / a.NS) & 1);
  }
}

// ---------------------------------------------------------------------------
// Host plan
// ---------------------------------------------------------------------------
struct Plan {
  Args a;
  int threads, grid;
  size_t smem;
};

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Smallest multiple of 16 bytes >= v with pitch % mod == rem.
static int64_t pitch_at(int64_t v, int mod, int rem) {
  int64_t p = round_up(v, 16);
  while (p % mod != rem) p += 16;
  return p;
}

// Row pitch of a stage's codes: rows one warp-wide shared-memory read touches
// (8, 4 or 2 of them, by the read width) land on distinct banks.
static int64_t code_pitch(int64_t row_bytes, int bits, int G) {
  const int nwd = bits == 4 ? G / 32 : bits == 8 ? G / 16 : (G >= 64 ? G / 64 : 1);
  if ((bits == 2 && G == 32) || nwd == 1 || nwd == 8) return pitch_at(row_bytes, 32, 16);
  if (nwd == 2) return pitch_at(row_bytes, 64, 32);
  return pitch_at(row_bytes, 128, 64);
}

// Shared-memory layout of a launch (ring depth, consumer warps, offsets) for
// staged activations of tok_stride bytes per token, tables of Gn groups and
// `parts` partials per tile (the largest over the matmuls of a sequence);
// the grid: one CTA per SM, each owning at least one 16-row tile of the
// smallest matmul (min_rows rows).
static bool place(Plan &pl, int64_t M, int U, int64_t tok_stride, int64_t Gn, int parts, bool dual, int sms,
                  int64_t min_rows) {
  Args &a = pl.a;
  const int MP = pow2_tokens(static_cast<int>(M));
  const int64_t budget = dual ? kDualSmem : 227 * 1024;
  const int max_w = dual ? kDualConsumers : kMaxConsumers;
  struct Layout {
    int64_t xs_off, zero_off, tab_off, red_off, bar_off, total;
  };
  auto layout = [&](int ns) {
    Layout L;
    int64_t off = static_cast<int64_t>(ns) * a.stage_bytes;
    L.xs_off = off;
    off += M * tok_stride;
    L.zero_off = round_up(off, 128) + 64;
    off = L.zero_off + a.zero_stride + U * 64;
    L.tab_off = round_up(off, 16);
    off = L.tab_off + static_cast<int64_t>(MP) * Gn * 16;
    L.red_off = off;
    off += static_cast<int64_t>(a.red_bufs) * parts * kRows * MP * 4;
    L.bar_off = round_up(off, 8);
    L.total = L.bar_off + (2 * ns + 2) * 8 + (2 * a.red_bufs + 3) * 4;
    return L;
  };
  // consumer warps: a divisor of NS * nper, so the units one warp takes in a
  // ring slot are consecutive phases of that slot's barriers (a warp never
  // waits on a phase two ahead of the barrier's).  Take the depth that fits and
  // allows the most consumers (then the deepest).
  const int nper = a.nper;
  auto consumers = [&](int ns) {
    for (int w = max_w; w >= 1; --w)
      if ((ns * nper) % w == 0) return w;
    return 1;
  };
  int best_ns = 0;
  for (int ns = 2; ns <= kMaxStages; ++ns) {
    if (layout(ns).total > budget) break;
    if (best_ns == 0 || consumers(ns) >= consumers(best_ns)) best_ns = ns;
  }
  if (best_ns == 0 || (dual && best_ns < kDualMinStages)) return false;
  const Layout L = layout(best_ns);
  a.NS = best_ns;
  a.W = consumers(best_ns);
  a.xs_off = static_cast<int>(L.xs_off);
  a.zero_off = static_cast<int>(L.zero_off);
  a.tab_off = static_cast<int>(L.tab_off);
  a.red_off = static_cast<int>(L.red_off);
  a.bar_off = static_cast<int>(L.bar_off);
  pl.smem = static_cast<size_t>(L.total);
  pl.threads = 32 * (a.W + 1);
  pl.grid = static_cast<int>(std::min<int64_t>(sms, min_rows / kRows));
  return true;
}

// fmt 0: affine codes with fp16 scales and biases; fmt 1: mxfp4 (E2M1 codes,
// one E8M0 byte per 32, no biases); fmt 2: nvfp4 (E2M1 codes, one E4M3 byte per
// 16, i.e. two per 32-code span, a tensor scale, no biases; M <= 4).
// dual: the plan for two CTAs per SM (this kernel's and the next launch's, when
// that one is a programmatic dependent): at most kDualSmem bytes of shared
// memory and kDualConsumers consumer warps, at least kDualMinStages stages.
// Codes of a row per work unit, for M tokens and nch K chunks per tile.  Units
// smaller than a stage spread a CTA's last stages over more warps (a shorter
// tail after the stream ends) and balance a CTA's few stages over its
// consumer warps, at the price of more partial sums per tile.  Measured on
// B200 (4-bit G64, decode chains): 1024-code units against whole stages of
// 2048 took the Llama-3-8B decode step from 28.3 to 27.9 us and the small-M
// curves up by 7-37% (M = 2..8, K = 4096 and 14336), except one token over
// seven chunks per tile (K = 14336: 11.6 -> 11.9 us), which keeps whole stages.
static int64_t unit_codes(int64_t M, int64_t nch) {
  if (M == 1 && nch > 4) return kUnitCodes;
  return AQ_QMV_SMALL_UNIT;
}

static bool make_plan_uncached(int64_t M, int64_t N, int64_t K, int G, int bits, int sms, Plan &pl, int fmt,
                               bool dual, int stage_target, int64_t unit_limit) {
  if (!(bits == 2 || bits == 4 || bits == 8) || !(G == 32 || G == 64 || G == 128)) return false;
  if (M < 1 || M > 8 || N < 1 || K < 1 || K % (8 * G) != 0) return false;
  // mxfp4 scale rows are K/32 bytes: a TMA row stride must be a multiple of 16 bytes
  if (fmt == 1 && (bits != 4 || G != 32 || K % 512 != 0)) return false;
  // nvfp4 scale rows are K/16 bytes
  if (fmt == 2 && (bits != 4 || G != 32 || K % 256 != 0 || M > 4)) return false;
  // mxfp8: 8-bit codes, scale rows of K/32 bytes as for mxfp4
  if (fmt == 3 && (bits != 8 || G != 32 || K % 512 != 0)) return false;
  if (N >= (int64_t(1) << 31) || K >= (int64_t(1) << 30)) return false;
  if (N < kRows) return false;  // every CTA owns at least one whole 16-row tile
  const int MP = pow2_tokens(static_cast<int>(M));
  const int64_t Gn = K / G, units = K / (8 * G);
  const int U = G / 32;
  // K chunk: the largest multiple u of 8 groups dividing K whose 16-row stage
  // of codes stays within the target
  int64_t u = 1;
  // (mxfp4: an even number of units, so that every chunk's scale box starts on
  // a 16-byte boundary: a chunk holds 8u scale bytes)
  const bool even_units = fmt == 1 || fmt == 3;
  if (even_units) u = 2;
  for (int64_t c = 1; c <= units; ++c)
    if (units % c == 0 && kRows * 8 * G * c * bits / 8 <= stage_target && (!even_units || c % 2 == 0)) u = c;
  const int64_t Kc = 8 * G * u, nch = K / Kc, gpc = Kc / G;
  Args &a = pl.a;
  a.njobs = 1;
  a.gbar = nullptr;
  a.experts = nullptr;
  a.E = 1;
  a.cta_per_tok = 0;
  a.gscale = nullptr;
  a.M = static_cast<int>(M);
  a.job[0].N = static_cast<int>(N);
  a.job[0].K = static_cast<int>(K);
  a.job[0].Gn = static_cast<int>(Gn);
  a.job[0].Kc = static_cast<int>(Kc);
  a.job[0].nch = static_cast<int>(nch);
  a.job[0].pitch_w = static_cast<int>(code_pitch(Kc * bits / 8, bits, G));
  const int sbytes = (fmt == 1 || fmt == 3) ? 1 : 2;  // scale bytes per 32-code span (nvfp4: two E4M3 bytes)
  a.job[0].pitch_s = static_cast<int>(pitch_at(gpc * sbytes, 32, 16));
  if (a.job[0].pitch_w / 8 > 256 || a.job[0].pitch_s / 8 > 256) return false;  // TMA box width (64-bit elements)
  a.job[0].w_box_x = static_cast<int>(Kc * bits / 64);
  a.job[0].sb_box_x = static_cast<int>(gpc * sbytes / 8);
  // every tiled TMA copy starts on a 16-byte boundary: x * 8 bytes % 16 == 0 for every chunk
  if (nch > 1 && (a.job[0].w_box_x % 2 != 0 || a.job[0].sb_box_x % 2 != 0)) return false;
  a.job[0].s_off = kRows * a.job[0].pitch_w;
  a.job[0].b_off = a.job[0].s_off + kRows * a.job[0].pitch_s;
  a.stage_bytes = static_cast<int>(round_up((fmt >= 1 ? a.job[0].s_off : a.job[0].b_off) + kRows * a.job[0].pitch_s, 128));
  a.job[0].tok_stride = static_cast<int>(2 * K + 64);
  a.zero_stride = static_cast<int>(round_up(U * 64, 128) + 64);
  // work units: fpu folds (a fold: the groups side by side above; nvfp4: twice as
  // many 16-weight groups) of one stage, at most unit_codes(M, nch) codes of a
  // row.  Every unit costs a partial-sum reduction (measured: units of 512
  // codes were 17% slower than whole stages on the 33 MB decode launches)
  // (a fold: the affine format holds 4/MP groups side by side, or one for
  // MP = 8; the block-scaled formats 8/MP)
  const int GS = 8 / MP, SPANS = fmt == 0 ? (MP >= 4 ? 1 : 4 / MP) : fmt == 2 ? GS / 2 : GS;
  const int64_t fold = static_cast<int64_t>(SPANS) * G;  // codes of a row per fold
  // folds per unit: the largest divisor of the stage's folds within kUnitCodes
  const int64_t stage_folds = Kc / fold;
  const int64_t ucodes = unit_limit > 0 ? unit_limit : unit_codes(M, nch);
  a.job[0].fpu = 1;
  for (int64_t d = 1; d <= stage_folds; ++d)
    if (stage_folds % d == 0 && fold * d <= ucodes) a.job[0].fpu = static_cast<int>(d);
  a.nper = static_cast<int>(Kc / (fold * a.job[0].fpu));
  a.job[0].parts = static_cast<int>(nch) * a.nper;
  // tiles in flight: the units in progress (one per warp, at most
  // kMaxConsumers) span at most two tiles once a tile has that many units
  a.red_bufs = a.job[0].parts == 1 ? 1 : a.job[0].parts >= 2 * kMaxConsumers ? 2 : a.job[0].parts >= kMaxConsumers ? 3 : kRedBufs;
  a.wait_cycles = kWaitCycles;
  a.stall = 0;
  return place(pl, M, U, a.job[0].tok_stride, Gn, a.job[0].parts, dual, sms, N);
}

// A plan is a function of its arguments alone, and one decode call computes the
// same plan several times (dispatch, validation, the launch): keep the last
// few per thread.
static bool make_plan(int64_t M, int64_t N, int64_t K, int G, int bits, int sms, Plan &pl, int fmt = 0,
                      bool dual = false, int stage_target = kStageTarget, int64_t unit_limit = 0) {
  struct Entry {
    int64_t M, N, K, unit_limit;
    int G, bits, sms, fmt, stage_target;
    bool dual, used, ok;
    Plan pl;
  };
  constexpr int kEntries = 8;
  static thread_local Entry cache[kEntries];
  static thread_local int next = 0;
  for (Entry &c : cache)
    if (c.used && c.M == M && c.N == N && c.K == K && c.unit_limit == unit_limit && c.G == G && c.bits == bits &&
        c.sms == sms && c.fmt == fmt && c.stage_target == stage_target && c.dual == dual) {
      if (c.ok) pl = c.pl;
      return c.ok;
    }
  Entry &c = cache[next];
  next = (next + 1) % kEntries;
  c.M = M; c.N = N; c.K = K; c.unit_limit = unit_limit;
  c.G = G; c.bits = bits; c.sms = sms; c.fmt = fmt; c.stage_target = stage_target; c.dual = dual;
  c.ok = make_plan_uncached(M, N, K, G, bits, sms, c.pl, fmt, dual, stage_target, unit_limit);
  c.used = true;
  if (c.ok) pl = c.pl;
  return c.ok;
}
using Maps = JobMaps<1>;

// The two-CTAs-per-SM plan for a call (the next launch's CTA beside this
// one's, so that its prologue and first copies overlap this launch's tail).
// Not used: it was slower on the decode step (37.4 against 26.7 us; only the
// 4096 x 4096 linear gained), and a small-M sweep with it did not finish within
// five minutes, consistent with its bounded waits running out on every launch.
// The launch path keeps the parameter for it.
static const Plan *dual_plan(const Plan &, bool, int64_t, int64_t, int64_t, int, int, int, int, Plan &) {
  return nullptr;
}

// Limit of the kernel's bounded waits, in SM clock cycles (aq_set_wait_limit).
static std::atomic<long long> g_wait_limit{kWaitCycles};
static std::atomic<bool> g_wait_stall{false};  // aq_set_wait_stall

// Registers per thread of a kernel instantiation (cached per thread and device).
template <int BITS, int G, int MP, int FMT>
static int kernel_regs() {
  static thread_local int cached_dev = -1, regs = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1 << 20;
  if (dev != cached_dev) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, qmv_tc_kernel<BITS, G, MP, FMT>) != cudaSuccess) return 1 << 20;
    regs = fa.numRegs;
    cached_dev = dev;
  }
  return regs;
}

// pl: the plan for one CTA per SM; dual (may be null): the plan for two per SM,
// used when the kernel's registers allow two such CTAs on an SM.  With a dual
// plan and overlap, every stage of the ring is issued before the kernel waits
// for the one before it: its CTAs run beside that kernel's, so the weights
// stream while the previous kernel finishes.
template <int BITS, int G, int MP, int FMT>
static cudaError_t launch(const Plan &pl_one, const Plan *dual, const Maps &mp, bool overlap, cudaStream_t stream) {
  auto kern = qmv_tc_kernel<BITS, G, MP, FMT>;
  const Plan *use = &pl_one;
  if (dual != nullptr) {
    const int regs = (kernel_regs<BITS, G, MP, FMT>() + 7) / 8 * 8;
    if (2 * regs * dual->threads <= 65536) use = dual;
  }
  Plan pl = *use;
  pl.a.wait_cycles = g_wait_limit.load(std::memory_order_relaxed);
  pl.a.stall = g_wait_stall.load(std::memory_order_relaxed) ? 1 : 0;
  static thread_local int cached_dev = -1;
  static thread_local size_t cached_smem = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev || pl.smem > cached_smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem))) !=
        cudaSuccess)
      return e;
    cached_dev = dev;
    cached_smem = pl.smem;
  }
  if (!overlap) {
    kern<<<pl.grid, pl.threads, pl.smem, stream>>>(pl.a, mp);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, pl.a, mp);
}

template <int BITS, int G, int FMT = 0>
static cudaError_t launch_mp(const Plan &pl, const Plan *dual, const Maps &mp, bool overlap, cudaStream_t stream) {
  switch (pow2_tokens(pl.a.M)) {
    case 1: return launch<BITS, G, 1, FMT>(pl, dual, mp, overlap, stream);
    case 2: return launch<BITS, G, 2, FMT>(pl, dual, mp, overlap, stream);
    case 4: return launch<BITS, G, 4, FMT>(pl, dual, mp, overlap, stream);
    default: return launch<BITS, G, 8, FMT>(pl, dual, mp, overlap, stream);
  }
}

template <int BITS>
static cudaError_t launch_g(const Plan &pl, const Plan *dual, const Maps &mp, int G, bool overlap,
                            cudaStream_t stream) {
  switch (G) {
    case 32: return launch_mp<BITS, 32>(pl, dual, mp, overlap, stream);
    case 64: return launch_mp<BITS, 64>(pl, dual, mp, overlap, stream);
    default: return launch_mp<BITS, 128>(pl, dual, mp, overlap, stream);
  }
}

// A [rows x row_bytes] row-major array as 64-bit elements, boxes of 16 rows x
// box_bytes (the stage pitch; columns past the end of a row read as zeros).
static bool encode_rows(CUtensorMap *map, const void *base, int64_t rows, int64_t row_bytes, int box_bytes) {
  auto fn = qmm::encode_fn();
  if (!fn) return false;
  return encode_2d_cached(fn, map, CU_TENSOR_MAP_DATA_TYPE_UINT64, base, static_cast<uint64_t>(row_bytes / 8),
                          static_cast<uint64_t>(rows), static_cast<uint64_t>(row_bytes),
                          static_cast<uint32_t>(box_bytes / 8), static_cast<uint32_t>(kRows),
                          CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ---------------------------------------------------------------------------
// Sequence launches: several matmuls (same M, G, bits) in one grid
// ---------------------------------------------------------------------------
// Grid barriers of sequence launches, one (count, generation) pair per slot.
// Consecutive launches take consecutive slots, so launches in flight at the
// same time on different streams share none unless kSeqBarSlots of them do.
constexpr int kSeqBarSlots = 64;
__device__ unsigned g_seq_bar[kSeqBarSlots][2];

static bool make_seq_plan(int n, const int64_t *N, const int64_t *K, int64_t M, int G, int bits, int sms, Plan &pl) {
  if (n < 1 || n > kSeqMax) return false;
  Plan pj[kSeqMax];
  for (int j = 0; j < n; ++j)  // (whole-stage units: one unit size for the whole ring)
    if (!make_plan(M, N[j], K[j], G, bits, sms, pj[j], 0, false, kStageTarget, kUnitCodes)) return false;
  pl = pj[0];
  Args &a = pl.a;
  a.njobs = n;
  int64_t tok = 0, gn = 0, rows = N[0];
  int parts = 0, stage = 0, red = 0;
  for (int j = 0; j < n; ++j) {
    if (pj[j].a.nper != a.nper) return false;  // one unit size for the whole ring
    a.job[j] = pj[j].a.job[0];
    tok = std::max<int64_t>(tok, a.job[j].tok_stride);
    gn = std::max<int64_t>(gn, a.job[j].Gn);
    parts = std::max(parts, a.job[j].parts);
    stage = std::max(stage, pj[j].a.stage_bytes);
    red = std::max(red, pj[j].a.red_bufs);
    rows = std::min(rows, N[j]);
  }
  a.stage_bytes = stage;
  a.red_bufs = red;
  return place(pl, M, G / 32, tok, gn, parts, false, sms, rows);
}

template <int BITS, int G, int MP>
static cudaError_t launch_seq(const Plan &pl_in, const JobMaps<kSeqMax> &mp, bool overlap, cudaStream_t stream) {
  auto kern = qmv_tc_kernel<BITS, G, MP, 0, kSeqMax>;
  Plan pl = pl_in;
  pl.a.wait_cycles = g_wait_limit.load(std::memory_order_relaxed);
  pl.a.stall = g_wait_stall.load(std::memory_order_relaxed) ? 1 : 0;
  static thread_local int cached_dev = -1;
  static thread_local size_t cached_smem = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev || pl.smem > cached_smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem))) !=
        cudaSuccess)
      return e;
    cached_dev = dev;
    cached_smem = pl.smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, pl.a, mp);
}

template <int BITS, int G>
static cudaError_t launch_seq_mp(const Plan &pl, const JobMaps<kSeqMax> &mp, bool overlap, cudaStream_t stream) {
  switch (pow2_tokens(pl.a.M)) {
    case 1: return launch_seq<BITS, G, 1>(pl, mp, overlap, stream);
    case 2: return launch_seq<BITS, G, 2>(pl, mp, overlap, stream);
    case 4: return launch_seq<BITS, G, 4>(pl, mp, overlap, stream);
    default: return launch_seq<BITS, G, 8>(pl, mp, overlap, stream);
  }
}

template <int BITS>
static cudaError_t launch_seq_g(const Plan &pl, const JobMaps<kSeqMax> &mp, int G, bool overlap, cudaStream_t stream) {
  switch (G) {
    case 32: return launch_seq_mp<BITS, 32>(pl, mp, overlap, stream);
    case 64: return launch_seq_mp<BITS, 64>(pl, mp, overlap, stream);
    default: return launch_seq_mp<BITS, 128>(pl, mp, overlap, stream);
  }
}

}  // namespace tc

bool qmv_tc_supported(int64_t M, int64_t N, int64_t K, int G, int bits) {
  tc::Plan pl;
  return tc::make_plan(M, N, K, G, bits, 148, pl);
}

cudaError_t launch_qmv_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                          const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, uint32_t flags,
                          cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  tc::Plan pl;
  if (!tc::make_plan(M, N, K, G, bits, sms, pl)) return cudaErrorInvalidValue;
  pl.a.job[0].x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.job[0].y = reinterpret_cast<__nv_bfloat16 *>(y);
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  tc::Plan dpl;
  const tc::Plan *dual = tc::dual_plan(pl, overlap, M, N, K, G, bits, sms, 0, dpl);
  tc::Maps mp;
  const int64_t row_bytes = K * bits / 8, sb_bytes = K / G * 2;
  if (!tc::encode_rows(&mp.w[0], packed, N, row_bytes, pl.a.job[0].pitch_w) ||
      !tc::encode_rows(&mp.s[0], scales, N, sb_bytes, pl.a.job[0].pitch_s) ||
      !tc::encode_rows(&mp.b[0], biases, N, sb_bytes, pl.a.job[0].pitch_s))
    return cudaErrorInvalidValue;
  switch (bits) {
    case 2: return tc::launch_g<2>(pl, dual, mp, G, overlap, s);
    case 4: return tc::launch_g<4>(pl, dual, mp, G, overlap, s);
    default: return tc::launch_g<8>(pl, dual, mp, G, overlap, s);
  }
}

bool qmv_tc_seq_supported(int n, const int64_t *N, const int64_t *K, int64_t M, int G, int bits) {
  tc::Plan pl;
  return tc::make_seq_plan(n, N, K, M, G, bits, 148, pl);
}

cudaError_t launch_qmv_tc_seq(int n, const SeqCall *calls, int64_t M, int G, int bits, uint32_t flags, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  if (n < 1 || n > tc::kSeqMax) return cudaErrorInvalidValue;
  int64_t N[tc::kSeqMax], K[tc::kSeqMax];
  for (int j = 0; j < n; ++j) {
    N[j] = calls[j].N;
    K[j] = calls[j].K;
  }
  tc::Plan pl;
  if (!tc::make_seq_plan(n, N, K, M, G, bits, sms, pl)) return cudaErrorInvalidValue;
  tc::JobMaps<tc::kSeqMax> mp;
  for (int j = 0; j < n; ++j) {
    pl.a.job[j].x = reinterpret_cast<const __nv_bfloat16 *>(calls[j].x);
    pl.a.job[j].y = reinterpret_cast<__nv_bfloat16 *>(calls[j].y);
    const int64_t row_bytes = K[j] * bits / 8, sb_bytes = K[j] / G * 2;
    if (!tc::encode_rows(&mp.w[j], calls[j].packed, N[j], row_bytes, pl.a.job[j].pitch_w) ||
        !tc::encode_rows(&mp.s[j], calls[j].scales, N[j], sb_bytes, pl.a.job[j].pitch_s) ||
        !tc::encode_rows(&mp.b[j], calls[j].biases, N[j], sb_bytes, pl.a.job[j].pitch_s))
      return cudaErrorInvalidValue;
  }
  for (int j = n; j < tc::kSeqMax; ++j) {  // unused entries: copies of the first (never read)
    mp.w[j] = mp.w[0];
    mp.s[j] = mp.s[0];
    mp.b[j] = mp.b[0];
  }
  // a grid barrier slot for this launch
  static std::atomic<unsigned> next_slot{0};
  void *bar = nullptr;
  if ((e = cudaGetSymbolAddress(&bar, tc::g_seq_bar)) != cudaSuccess) return e;
  const unsigned slot = next_slot.fetch_add(1, std::memory_order_relaxed) % tc::kSeqBarSlots;
  pl.a.gbar = reinterpret_cast<unsigned *>(bar) + 2 * slot;
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  switch (bits) {
    case 2: return tc::launch_seq_g<2>(pl, mp, G, overlap, s);
    case 4: return tc::launch_seq_g<4>(pl, mp, G, overlap, s);
    default: return tc::launch_seq_g<8>(pl, mp, G, overlap, s);
  }
}

cudaError_t launch_gather_tc(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed, const uint16_t *scales,
                             const uint16_t *biases, int64_t E, int64_t N, int G, int bits, const int32_t *experts,
                             uint16_t *y, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  tc::Plan pl;
  if (!tc::make_plan(1, N, K, G, bits, sms, pl)) return cudaErrorInvalidValue;
  // CTAs per token: the SMs shared out between the tokens, each CTA >= 16 rows
  const int64_t per_tok = std::max<int64_t>(1, std::min<int64_t>(sms / std::max<int64_t>(T, 1), N / tc::kRows));
  if (T * per_tok >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  pl.grid = static_cast<int>(T * per_tok);
  pl.a.cta_per_tok = static_cast<int>(per_tok);
  pl.a.experts = experts;
  pl.a.E = static_cast<int>(E);
  pl.a.job[0].x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.job[0].y = reinterpret_cast<__nv_bfloat16 *>(y);
  tc::Maps mp;
  const int64_t row_bytes = K * bits / 8, sb_bytes = K / G * 2;
  if (!tc::encode_rows(&mp.w[0], packed, E * N, row_bytes, pl.a.job[0].pitch_w) ||
      !tc::encode_rows(&mp.s[0], scales, E * N, sb_bytes, pl.a.job[0].pitch_s) ||
      !tc::encode_rows(&mp.b[0], biases, E * N, sb_bytes, pl.a.job[0].pitch_s))
    return cudaErrorInvalidValue;
  switch (bits) {
    case 2: return tc::launch_g<2>(pl, nullptr, mp, G, false, s);
    case 4: return tc::launch_g<4>(pl, nullptr, mp, G, false, s);
    default: return tc::launch_g<8>(pl, nullptr, mp, G, false, s);
  }
}

bool mxfp4_tc_supported(int64_t M, int64_t N, int64_t K) {
  tc::Plan pl;
  return tc::make_plan(M, N, K, 32, 4, 148, pl, 1);
}

// mxfp4 (E2M1 codes packed 8 per word, one E8M0 scale byte per 32 along K).
cudaError_t launch_mxfp4_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  tc::Plan pl;
  if (!tc::make_plan(M, N, K, 32, 4, sms, pl, 1)) return cudaErrorInvalidValue;
  pl.a.job[0].x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.job[0].y = reinterpret_cast<__nv_bfloat16 *>(y);
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  tc::Plan dpl;
  const tc::Plan *dual = tc::dual_plan(pl, overlap, M, N, K, 32, 4, sms, 1, dpl);
  tc::Maps mp;
  if (!tc::encode_rows(&mp.w[0], packed, N, K / 2, pl.a.job[0].pitch_w) || !tc::encode_rows(&mp.s[0], scales, N, K / 32, pl.a.job[0].pitch_s))
    return cudaErrorInvalidValue;
  mp.b[0] = mp.s[0];  // no bias map: the kernel never reads this one
  return tc::launch_mp<4, 32, 1>(pl, dual, mp, overlap, s);
}

bool mxfp8_tc_supported(int64_t M, int64_t N, int64_t K) {
  tc::Plan pl;
  return tc::make_plan(M, N, K, 32, 8, 148, pl, 3);
}

// mxfp8 (E4M3 codes packed 4 per word, one E8M0 byte per 32 along K).
cudaError_t launch_mxfp8_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  tc::Plan pl;
  if (!tc::make_plan(M, N, K, 32, 8, sms, pl, 3)) return cudaErrorInvalidValue;
  pl.a.job[0].x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.job[0].y = reinterpret_cast<__nv_bfloat16 *>(y);
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  tc::Plan dpl;
  const tc::Plan *dual = tc::dual_plan(pl, overlap, M, N, K, 32, 8, sms, 3, dpl);
  tc::Maps mp;
  if (!tc::encode_rows(&mp.w[0], packed, N, K, pl.a.job[0].pitch_w) || !tc::encode_rows(&mp.s[0], scales, N, K / 32, pl.a.job[0].pitch_s))
    return cudaErrorInvalidValue;
  mp.b[0] = mp.s[0];  // no bias map: the kernel never reads this one
  return tc::launch_mp<8, 32, 3>(pl, dual, mp, overlap, s);
}

bool nvfp4_tc_supported(int64_t M, int64_t N, int64_t K) {
  tc::Plan pl;
  return tc::make_plan(M, N, K, 32, 4, 148, pl, 2);
}

// nvfp4 (E2M1 codes packed 8 per word, one E4M3 byte per 16 along K, the fp32
// tensor scale at gscale on the device).
cudaError_t launch_nvfp4_tc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *scales,
                            const float *gscale, int64_t N, uint16_t *y, uint32_t flags, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  tc::Plan pl;
  if (!tc::make_plan(M, N, K, 32, 4, sms, pl, 2)) return cudaErrorInvalidValue;
  pl.a.job[0].x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.gscale = gscale;
  pl.a.job[0].y = reinterpret_cast<__nv_bfloat16 *>(y);
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  tc::Plan dpl;
  const tc::Plan *dual = tc::dual_plan(pl, overlap, M, N, K, 32, 4, sms, 2, dpl);
  tc::Maps mp;
  if (!tc::encode_rows(&mp.w[0], packed, N, K / 2, pl.a.job[0].pitch_w) || !tc::encode_rows(&mp.s[0], scales, N, K / 16, pl.a.job[0].pitch_s))
    return cudaErrorInvalidValue;
  mp.b[0] = mp.s[0];  // no bias map: the kernel never reads this one
  switch (tc::pow2_tokens(pl.a.M)) {
    case 1: return tc::launch<4, 32, 1, 2>(pl, dual, mp, overlap, s);
    case 2: return tc::launch<4, 32, 2, 2>(pl, dual, mp, overlap, s);
    default: return tc::launch<4, 32, 4, 2>(pl, dual, mp, overlap, s);
  }
}

void set_qmv_tc_wait_limit(long long cycles) { tc::g_wait_limit.store(cycles > 0 ? cycles : kWaitCycles); }
void set_qmv_tc_wait_stall(bool on) { tc::g_wait_stall.store(on); }

cudaError_t read_and_clear_qmv_tc_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_qmv_tc_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  if (*word != 0) {
    // a sequence launch that gave up may have left a grid barrier half passed
    static const unsigned zeros[tc::kSeqBarSlots][2] = {};
    if ((e = cudaMemcpyToSymbol(tc::g_seq_bar, zeros, sizeof(zeros))) != cudaSuccess) return e;
  }
  return cudaMemcpyToSymbol(g_qmv_tc_fault, &zero, sizeof(uint32_t));
}

}  // namespace aq
