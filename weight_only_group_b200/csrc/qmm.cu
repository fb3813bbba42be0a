// QMM: quantized matrix x matrix for prefill on the 5th-generation tensor
// cores (tcgen05 + tensor memory), sm_100a.
//
// Method: metalworking "MLX Quantization", section "Mechanics": QMM is the
// prefill/batch case: dequantize weight tiles on chip, then a tiled GEMM
// against them; "One trap for intuition": dequantize on every use, never a
// cached fp16 copy.  anllm "Tutorial 10: Quantization", section 5: the fused
// product equals dequantize-then-multiply.
//
// Precision: both MMA operands are fp16 (11-bit significands).  Dequantized
// weights are fp16_rn(fp32_rn(q*scale + bias)); bf16 (8 bits) is not enough:
// in groups stretched by an outlier the bf16 rounding of every weight adds up
// past the matmul tolerance.  Activations are carried as fp16 after an exact
// power-of-two scaling of each token row (x = 2^e * x16, the row maximum of
// x16 in [2^14, 2^15)), done by a small pre-pass into workspace memory; the
// epilogue multiplies the fp32 accumulator by 2^e.
//
// B200 design ("swap AB": weights are the MMA's A operand, tokens its N):
//  * CTA tile: 128 rows of W (MMA M = 128, one TMEM lane per row) x BN tokens
//    (MMA N = BN <= 256); persistent CTAs walk the tiles, token tiles fastest.
//  * Warp 0 (one lane): TMA producer.  Per K block it loads the x16 tile
//    [BN tokens x BK] (fp16, 128-byte swizzle, the canonical K-major UMMA
//    layout) and the packed W tile [128 rows x BK*bits/32 words] into a ring
//    of shared-memory stages, completing on the stage's mbarrier.
//  * Warps 4..15 (three per TMEM lane quadrant): dequantize.  Thread (quadrant,
//    lane) owns W row 32*quadrant+lane; the quadrant's three warps take K
//    blocks in turn (each warp a whole block, so it has three MMA blocks of
//    time per block of dequantization; measured 852 against 829 TFLOP/s with
//    two): it reads
//    its packed words from shared memory, turns codes into fp16 weights in
//    registers and writes them with tcgen05.st straight into a TMEM stage
//    that the MMA reads as operand A (no swizzled shared-memory round trip).
//  * Warp 1 (one lane): issues tcgen05.mma.kind::f16 (fp16 A from TMEM, fp16 B from
//    shared memory, fp32 accumulator of 128 x BN in TMEM) and tcgen05.commit
//    to release stages; warp 1 also owns the TMEM allocation.
//  * Epilogue: the dequant warps read the accumulator with tcgen05.ld, scale
//    by 2^e of the token row and store bf16 (RNE) y[m, n] (a warp writes 32
//    consecutive n per token).
//  * Every mbarrier wait is bounded; on expiry the kernel records a bit in a
//    device fault word, stops issuing work and exits cleanly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc05.cuh"

namespace aq {

__device__ uint32_t g_fault_word = 0;

namespace qmm {

constexpr int kDequantPerQuadrant = 3;
// Turns of scale / bias loads a dequant warp keeps in flight (a register queue
// with static indices; 4 was slower than 2, measured).  These loads hit L1:
// shared memory left unused by a kernel is L1 on this part, and every 24 KB
// more shared memory per CTA cost ~5-25% at K = 14336 (measured), so the
// kernels keep their shared memory tight.
constexpr int kSbAhead = 2;  // dequant warps per TMEM lane quadrant; they take turns on K blocks
constexpr int kDequantWarp0 = 4;        // warps 4.. dequantize + epilogue
constexpr int kThreads = 32 * (kDequantWarp0 + 4 * kDequantPerQuadrant);
constexpr int kTmemCols = 512;
constexpr int kAccCol = 0;        // accumulator columns [0, BN); A stages follow from column BN

// ---------------------------------------------------------------------------
// PTX wrappers: tc05.cuh
// ---------------------------------------------------------------------------
// Bounded wait on this kernel's fault word.
AQ_DEVICE bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t fault_bit) {
  return aq::mbar_wait(bar, parity, abort_flag, &g_fault_word, fault_bit);
}


// ---------------------------------------------------------------------------
// Tile configuration
// ---------------------------------------------------------------------------
constexpr int kGroupMaxE = 256;  // experts of a grouped launch at most (their tables live in shared memory)
constexpr int kGroupTabBytes = (2 * kGroupMaxE + 4) * 4;

template <int BITS, int BN>
struct Cfg {
  static constexpr int BK = (BITS == 3) ? 128 : 64;         // K per stage (elements)
  static constexpr int BKW = BK * BITS / 32;                // packed words per W row per stage
  static constexpr int X_BYTES = BN * BK * 2;               // x tile bytes
  static constexpr int W_BYTES = 128 * BKW * 4;             // packed W tile bytes
  static constexpr int STAGE_BYTES = ((X_BYTES + W_BYTES + 1023) / 1024) * 1024;
  static constexpr int SMEM_BUDGET = 225 * 1024;
  static constexpr int A_COLS = BK / 2;                     // TMEM columns per A stage (2 bf16 per column)
  static constexpr int A_COL0 = BN;                         // first TMEM column of the A stages
  static constexpr int STAGES = std::min(std::min(6, SMEM_BUDGET / STAGE_BYTES), (kTmemCols - A_COL0) / A_COLS);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ + kGroupTabBytes;
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  static_assert(A_COL0 + STAGES * A_COLS <= kTmemCols, "TMEM budget");
  static_assert(BN <= 256 && BN % 16 == 0, "MMA N");
};

// Dequantization into TMEM columns and the K interleave of x16: tc05.cuh.

struct Params {
  const __half *scales;
  const __half *biases;
  const float *row_scale;  // per token row: x[m,:] = row_scale[m] * x16[m,:] exactly
  __nv_bfloat16 *y;
  int M, N, K, G, Gn;
  int m_tiles, n_tiles;
  int n_fastest;  // tile order: W-row tiles fastest (else token tiles fastest)
  // grouped mode (E experts > 0): the M token rows are E consecutive segments,
  // segment e = rows [offsets[e], offsets[e+1]) multiplied by expert e (rows
  // e*N .. e*N+N-1 of the stacked W); offsets live in device memory
  const int32_t *offsets;
  int E;
  // block-scaled formats: one scale byte per 32 codes (mxfp4 / mxfp8, E8M0) or
  // per 16 (nvfp4, E4M3) in rows of sb_row bytes, and nvfp4's tensor scale
  const uint8_t *bscales;
  int sb_row;
  const float *gscale;
  // K split of the CTA-pair kernel: each tile's K blocks are cut into ksplit
  // contiguous parts, one work item each (tile w % tiles, part w / tiles for
  // item w).  Every part writes its fp32 sums to `partial`; the part that
  // arrives last on the tile's counters (`arrivals`, zeroed by the pre-pass)
  // adds the parts in part order and writes y.
  int ksplit = 1;
  float *partial = nullptr;
  uint32_t *arrivals = nullptr;
};

// Largest byte of a row of n scale bytes (E8M0 and positive E4M3 order like
// their bits): 16-byte loads where the row allows them, single bytes otherwise
// (rows of K/32 bytes start on 16-byte boundaries only when K % 512 == 0).
AQ_DEVICE uint32_t row_max_byte(const uint8_t *row, int n) {
  uint32_t mx = 0;
  if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0 && (n & 15) == 0) {
    for (int i = 0; i < n / 16; ++i) {
      const uint4 v = ldg_nc16(row + 16 * i);
      mx = __vmaxu4(mx, __vmaxu4(__vmaxu4(v.x, v.y), __vmaxu4(v.z, v.w)));
    }
    return max(max(mx & 0xFFu, (mx >> 8) & 0xFFu), max((mx >> 16) & 0xFFu, mx >> 24));
  }
  for (int i = 0; i < n; ++i) mx = max(mx, static_cast<uint32_t>(__ldg(row + i)));
  return mx;
}

// One tile of a launch: its first token row and first W row in the maps, the
// W row within the weight matrix (or expert), and the end of its token rows.
struct TileRef {
  int m0, n0, wrow, mend;
};

// Tile t's first token and first W row.  Token tiles fastest keeps a W tile in
// use by many CTAs at once (the fp16 activations stay in L2); W-row tiles
// fastest keeps an activation tile in use instead, for activations that do not
// fit in L2.
// A tile is bn tokens x wr rows of W.
AQ_DEVICE void tile_origin(const Params &prm, int tile, int bn, int wr, int &m0, int &n0) {
  if (prm.n_fastest) {
    m0 = (tile / prm.n_tiles) * bn;
    n0 = (tile % prm.n_tiles) * wr;
  } else {
    m0 = (tile % prm.m_tiles) * bn;
    n0 = (tile / prm.m_tiles) * wr;
  }
}

// Tile t of a launch.  Grouped mode: tiles run over (segment tile, W tile)
// pairs, W tiles fastest; seg[] holds the E + 1 segment offsets and mtp[] the
// prefix sums of each segment's token tiles.
AQ_DEVICE TileRef tile_at(const Params &prm, const int *seg, const int *mtp, int tile, int bn) {
  TileRef r;
  if (prm.E == 0) {
    tile_origin(prm, tile, bn, 128, r.m0, r.n0);
    r.wrow = r.n0;
    r.mend = prm.M;
    return r;
  }
  const int nt = tile % prm.n_tiles, mg = tile / prm.n_tiles;
  int lo = 0, hi = prm.E - 1;  // the segment e with mtp[e] <= mg < mtp[e + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mtp[mid] <= mg) lo = mid; else hi = mid - 1;
  }
  r.m0 = seg[lo] + (mg - mtp[lo]) * bn;
  r.n0 = nt * 128;
  r.wrow = lo * prm.N + r.n0;
  r.mend = seg[lo + 1];
  return r;
}

// FMT: 0 affine (fp16 scale and bias per G codes); 1 mxfp4, 2 nvfp4, 3 mxfp8.
template <int BITS, int BN, int FMT = 0>
__global__ void __launch_bounds__(kThreads, 1) qmm_kernel(const __grid_constant__ CUtensorMap x_map,
                                                          const __grid_constant__ CUtensorMap w_map, Params prm) {
  using C = Cfg<BITS, BN>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);
  uint64_t *empty = full + S;
  uint64_t *a_full = empty + S;
  uint64_t *acc_full = a_full + S;
  uint64_t *acc_empty = acc_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *seg = reinterpret_cast<int *>(smem + S * C::STAGE_BYTES + 256);  // grouped: [E + 1] offsets
  int *mtp = seg + kGroupMaxE + 2;                                     // grouped: [E + 1] tile prefix sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = (prm.K + C::BK - 1) / C::BK;
  if (prm.E > 0 && threadIdx.x == 64) {  // warp 2 (otherwise idle) reads the segments
    int run = 0;
    for (int e = 0; e <= prm.E; ++e) {
      seg[e] = __ldg(prm.offsets + e);
      mtp[e] = run;
      if (e < prm.E) run += (__ldg(prm.offsets + e + 1) - seg[e] + BN - 1) / BN;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&a_full[s], 4);  // one warp per TMEM lane quadrant fills a K block
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4 * kDequantPerQuadrant);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = prm.E > 0 ? prm.n_tiles * mtp[prm.E] : prm.m_tiles * prm.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&x_map)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&w_map)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const TileRef tr = tile_at(prm, seg, mtp, tile, BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          if (r >= 1 && !(ok = mbar_wait(&empty[s], (r - 1) & 1, abort_flag, kFaultProducerWait))) break;
          uint8_t *xs = smem + s * C::STAGE_BYTES;
          uint8_t *ws = xs + C::X_BYTES;
          mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::W_BYTES);
#pragma unroll
          for (int a = 0; a < C::BK / 64; ++a)
            tma_load_2d(xs + a * BN * 128, &x_map, &full[s], kb * C::BK + a * 64, tr.m0);
          tma_load_2d(ws, &w_map, &full[s], kb * C::BKW, tr.wrow);
        }
      }
      // drain: wait (bounded) until every issued load has landed
      const uint32_t issued = it;
      for (uint32_t j = (issued > static_cast<uint32_t>(S) ? issued - S : 0); j < issued; ++j) {
        mbar_drain(&full[j % S], (j / S) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BN);
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t) {
        if (t >= 1 && !(ok = mbar_wait(acc_empty, (t - 1) & 1, abort_flag, kFaultMmaWait))) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          if (!(ok = mbar_wait(&full[s], r & 1, abort_flag, kFaultMmaWait))) break;
          if (!(ok = mbar_wait(&a_full[s], r & 1, abort_flag, kFaultMmaWait))) break;
          tc_fence_after();
          const uint32_t xs_addr = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t a_tmem = tmem_base + C::A_COL0 + s * C::A_COLS;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            // K = 16 slice kk: 32 bytes into a 128-byte swizzle row; a new atom column every 64 elements
            const uint32_t b_addr = xs_addr + (kk / 4) * BN * 128 + (kk % 4) * 32;
            tc_mma_ts(tmem_base + kAccCol, a_tmem + kk * 8, sw128_kmajor_desc(b_addr), idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(acc_full);
      }
      // drain: the last commits must have landed before TMEM is released
      if (it > 0) mbar_drain(&empty[(it - 1) % S], ((it - 1) / S) & 1);
    }
  } else if (warp >= kDequantWarp0) {
    // ------------------------------------------------------------------ dequant + epilogue
    const int q = warp & 3;                     // TMEM lane quadrant
    const int h = (warp - kDequantWarp0) >> 2;  // the warps of a quadrant take K blocks in turn
    constexpr int H = kDequantPerQuadrant;
    const int row = q * 32 + lane;              // W row within the tile == TMEM lane
    constexpr int CH = C::BK / 32;              // 32-code chunks per thread per K block
    uint32_t it0 = 0, t = 0;                    // stage counter at the start of the tile
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t, it0 += KB) {
      const TileRef tr = tile_at(prm, seg, mtp, tile, BN);
      const int m0 = tr.m0;
      const int n = tr.n0 + row;
      const bool row_ok = n < prm.N;
      const int64_t g_row = static_cast<int64_t>(row_ok ? tr.wrow + row : 0) * prm.Gn;
      // Block-scaled formats: this row's power of two 2^-B (from its largest
      // scale byte; positive E4M3 and E8M0 order like their bits) keeps every
      // dequantized value within fp16; the epilogue multiplies by 2^B.
      const uint8_t *sbrow = nullptr;
      int bexp = 0;
      float rowfac = 1.0f;
      if constexpr (FMT != 0) {
        sbrow = prm.bscales + static_cast<int64_t>(row_ok ? tr.wrow + row : 0) * prm.sb_row;
        const uint32_t mx = row_ok ? row_max_byte(sbrow, prm.sb_row) : 0u;
        if constexpr (FMT == 2) {
          const float vmax = e4m3_value(mx);
          bexp = vmax > 0.0f ? static_cast<int>((__float_as_uint(vmax) >> 23) & 0xFFu) - 127 + 1 - 13 : 0;
          rowfac = pow2f_exact(bexp) * __ldg(prm.gscale);
        } else {
          bexp = static_cast<int>(mx) - 127 - (FMT == 1 ? 13 : 7);
          rowfac = pow2f_exact(bexp);
        }
      }
      // scales/biases (fp16 bits; block-scaled: the chunk's scale bytes) of this
      // thread's chunks, prefetched for this warp's next two K blocks (its turns
      // come every H blocks)
      auto load_sb = [&](int kb, uint16_t (&sc)[CH], uint16_t (&bi)[CH]) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          if constexpr (FMT == 0) {
            const int g = (kb * C::BK + c * 32) / prm.G;
            const bool in = row_ok && kb < KB && g < prm.Gn;
            sc[c] = in ? ldg_nc2(prm.scales + g_row + g) : uint16_t(0);
            bi[c] = in ? ldg_nc2(prm.biases + g_row + g) : uint16_t(0);
          } else {
            const int g32 = (kb * C::BK + c * 32) / 32;  // the chunk's 32-code span
            const bool in = row_ok && kb < KB && g32 < prm.K / 32;
            sc[c] = !in ? uint16_t(0) : FMT == 2 ? ldg_nc2(sbrow + 2 * g32) : static_cast<uint16_t>(sbrow[g32]);
            bi[c] = 0;
          }
        }
      };
      // a queue of the next kSbAhead turns' scales, shifted by one each turn
      // (static indices keep it in registers)
      uint16_t sc_pf[kSbAhead][CH], bi_pf[kSbAhead][CH];
#pragma unroll
      for (int i = 0; i < kSbAhead; ++i) load_sb(h + i * H, sc_pf[i], bi_pf[i]);
      for (int kb = h; kb < KB; kb += H) {
        const uint32_t it = it0 + kb;
        const int s = it % S;
        const uint32_t r = it / S;
        uint16_t sc[CH], bi[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          sc[c] = sc_pf[0][c];
          bi[c] = bi_pf[0][c];
        }
#pragma unroll
        for (int i = 0; i + 1 < kSbAhead; ++i)
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            sc_pf[i][c] = sc_pf[i + 1][c];
            bi_pf[i][c] = bi_pf[i + 1][c];
          }
        load_sb(kb + kSbAhead * H, sc_pf[kSbAhead - 1], bi_pf[kSbAhead - 1]);
        if (!(ok = mbar_wait(&full[s], r & 1, abort_flag, kFaultDequantWait))) break;
        if (r >= 1 && !(ok = mbar_wait(&empty[s], (r - 1) & 1, abort_flag, kFaultDequantWait))) break;
        __syncwarp();  // lanes leave the spin at different times; tcgen05.st needs the whole warp
        const uint32_t *wrow =
            reinterpret_cast<const uint32_t *>(smem + s * C::STAGE_BYTES + C::X_BYTES) + row * C::BKW;
        const uint32_t a_tmem = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::A_COL0 + s * C::A_COLS;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          uint32_t w[BITS];
          if constexpr (BITS == 4) {
            const uint4 v4 = *reinterpret_cast<const uint4 *>(wrow + c * 4);
            w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
          } else if constexpr (BITS == 8) {
            const uint4 a4 = reinterpret_cast<const uint4 *>(wrow + c * 8)[0];
            const uint4 b4 = reinterpret_cast<const uint4 *>(wrow + c * 8)[1];
            w[0] = a4.x; w[1] = a4.y; w[2] = a4.z; w[3] = a4.w;
            w[4] = b4.x; w[5] = b4.y; w[6] = b4.z; w[7] = b4.w;
          } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) w[i] = wrow[c * BITS + i];
          }
          uint32_t packed_cols[16];
          if constexpr (FMT == 0) {
            dequant_chunk_f16<BITS>(w, sc[c], bi[c], packed_cols);
          } else if constexpr (FMT == 1) {
            const __half2 f = __float2half2_rn(pow2f_exact(static_cast<int>(sc[c]) - 127 - bexp));
            dequant_chunk_e2m1(reinterpret_cast<const uint32_t(&)[4]>(w), f, f, packed_cols);
          } else if constexpr (FMT == 2) {
            const float p2 = pow2f_exact(-bexp);
            const __half2 f0 = __float2half2_rn(e4m3_value(sc[c] & 0xFFu) * p2);
            const __half2 f1 = __float2half2_rn(e4m3_value(sc[c] >> 8) * p2);
            dequant_chunk_e2m1(reinterpret_cast<const uint32_t(&)[4]>(w), f0, f1, packed_cols);
          } else {
            const __half2 f = __float2half2_rn(pow2f_exact(static_cast<int>(sc[c]) - 127 - bexp + 8));
            dequant_chunk_e4m3(reinterpret_cast<const uint32_t(&)[8]>(w), f, packed_cols);
          }
          tmem_st16(a_tmem + c * 16, packed_cols);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[s]);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      if (!(ok = mbar_wait(acc_full, t & 1, abort_flag, kFaultEpilogueWait))) break;
      __syncwarp();
      tc_fence_after();
      // accumulator columns in blocks of 32, dealt round-robin to the quadrant's warps
#pragma unroll 1
      for (int col = h * 32; col < BN; col += H * 32) {
        uint32_t v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kAccCol + col, v);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int m = m0 + col + i;
            if (m < tr.mend)
              prm.y[static_cast<int64_t>(m) * prm.N + n] =
                  __float2bfloat16_rn(__uint_as_float(v[i]) * __ldg(prm.row_scale + m) * rowfac);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair kernel (tcgen05 cta_group::2).  Two CTAs of a cluster share one
// 256 x BN tile: CTA r owns W rows n0 + 128 r .. + 127 (its TMEM lanes, its A
// operand, its half of the accumulator) and tokens m0 + r BN/2 .. of the x16
// tile (its half of the B operand).  CTA 0 issues one M = 256 MMA per K = 16
// step for both; the tensor cores exchange the B halves.  Per K block a CTA
// thus stages BN/2 token rows instead of BN, which halves the shared-memory
// writes and the B reads per multiply-add and the L2 traffic behind them (the
// single-CTA kernel ran at about 800 cycles per 64-deep K block against 512
// of tensor work, with the stage ring unable to cover the load latency).
//   * both CTAs: TMA producer (warp 0) into their own stage ring, completing
//     on their own `full` barrier; dequant warps wait on it, write their A
//     stage into their own TMEM and arrive on CTA 0's `a_full` (eight
//     arrivals: four quadrant warps per CTA);
//   * CTA 0 warp 1: waits `a_full`, issues the pair MMAs, and commits with a
//     multicast arrive on both CTAs' `empty` (stage reuse) and `acc_full`;
//   * epilogue: each CTA reads its own accumulator rows, then arrives on CTA
//     0's `acc_empty` (24 arrivals).
// TMEM is allocated with cta_group::2 by warp 1 of both CTAs and freed after
// a cluster barrier that follows every MMA and every accumulator read.
// ---------------------------------------------------------------------------
template <int BITS, int BN>
struct PairCfg {
  static constexpr int BK = (BITS == 3) ? 128 : 64;
  static constexpr int BKW = BK * BITS / 32;
  static constexpr int XH = BN / 2;                          // token rows of the x16 tile in this CTA
  static constexpr int X_BYTES = XH * BK * 2;
  static constexpr int W_BYTES = 128 * BKW * 4;
  static constexpr int STAGE_BYTES = ((X_BYTES + W_BYTES + 1023) / 1024) * 1024;
  // epilogue staging: per dequant warp one 32 x 32 bf16 output box for TMA stores
  static constexpr int EPI_BYTES = 4 * kDequantPerQuadrant * 2048;
  static constexpr int SMEM_BUDGET = 225 * 1024 - EPI_BYTES;
  static constexpr int A_COLS = BK / 2;
  static constexpr int A_COL0 = BN;
  static constexpr int STAGES = std::min(std::min(12, SMEM_BUDGET / STAGE_BYTES), (kTmemCols - A_COL0) / A_COLS);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 512 /*barriers*/ + EPI_BYTES;
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  static_assert((3 * STAGES + 2) * 8 + 8 <= 512, "barrier area");
  static_assert(XH % 8 == 0 && BN <= 256 && BN % 32 == 0, "pair MMA N");
};

AQ_DEVICE uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
AQ_DEVICE void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the barrier at the same offset in CTA `cta` of the cluster.  The
// default (CTA-scope) release: a cluster-scope release would first wait for
// this thread's outstanding global loads (the scale prefetches), which put a
// full memory round trip into every K block.  What the arrive publishes is
// ordered by other means: tcgen05.st by wait::st and fence::before_thread_sync,
// the stage's TMA data by the barrier this thread waited on before.
AQ_DEVICE void mbar_arrive_at(uint64_t *bar, uint32_t cta) {
  uint32_t addr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(smem_u32(bar)), "r"(cta));
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
// Bounded wait on a barrier that the other CTA of the pair (or its tensor
// core commits) may complete.
AQ_DEVICE bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t fault_bit) {
  return mbar_wait(bar, parity, abort_flag, fault_bit);
}
AQ_DEVICE void tc_mma_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the MMAs issued so far have completed.
AQ_DEVICE void tc_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
// TMA store of a 2-D box from shared memory, in this thread's bulk group.
AQ_DEVICE void tma_store_2d(const CUtensorMap *map, const void *src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
AQ_DEVICE void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
AQ_DEVICE void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
AQ_DEVICE void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The work items of one CTA pair: items pair, pair + npairs, ... of the
// launch, item w being K part w / tiles of tile w % tiles.
struct PairItem {
  int tile, kb0, kb1;  // tile index (tile_origin) and its K blocks [kb0, kb1)
  int part;            // K part of the tile (0 .. ksplit - 1)
};
template <bool SPLIT>
struct PairCursor {
  uint32_t w, P, T, KB, ks;
  AQ_DEVICE PairCursor(const Params &prm, int pair, int npairs, int KB_, int tiles)
      : w(pair), P(npairs), T(tiles), KB(KB_), ks(SPLIT ? prm.ksplit : 1) {}
  AQ_DEVICE PairCursor(const Params &prm, int pair, int npairs, int KB_)
      : w(pair), P(npairs), T(prm.m_tiles * prm.n_tiles), KB(KB_), ks(SPLIT ? prm.ksplit : 1) {}
  AQ_DEVICE bool next(PairItem &it) {
    if constexpr (!SPLIT) {
      if (w >= T) return false;
      it.tile = static_cast<int>(w);
      it.part = 0;
      it.kb0 = 0;
      it.kb1 = static_cast<int>(KB);
      w += P;
      return true;
    }
    if (w >= T * ks) return false;
    const uint32_t part = w / T;
    it.tile = static_cast<int>(w - part * T);
    it.part = static_cast<int>(part);
    it.kb0 = static_cast<int>(part * KB / ks);  // (KB * ks < 2^32: the host caps ks at 4)
    it.kb1 = static_cast<int>((part + 1) * KB / ks);
    w += P;
    return true;
  }
};

// kind::f16 instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, M = 256, N = bn.
__host__ __device__ constexpr uint32_t idesc_pair(int bn) {
  return (1u << 4) | (static_cast<uint32_t>(bn >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
}

// SPLIT: the launch cuts tiles into K parts (Params::ksplit > 1).  FMT as in
// qmm_kernel: 0 affine, 1 mxfp4, 2 nvfp4, 3 mxfp8.
// GROUPED (affine, unsplit): the M token rows are E segments with device
// offsets (Params::offsets), segment e multiplied by expert e (rows e*N .. of
// the stacked W); token tiles of 256 never straddle a segment.
template <int BITS, int BN, bool SPLIT, int FMT = 0, bool GROUPED = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    qmm_pair_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap y_map, Params prm) {
  using C = PairCfg<BITS, BN>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);
  uint64_t *empty = full + S;
  uint64_t *a_full = empty + S;
  uint64_t *acc_full = a_full + S;
  uint64_t *acc_empty = acc_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int KB = (prm.K + C::BK - 1) / C::BK;
  static_assert(!GROUPED || (!SPLIT && FMT == 0), "grouped launches are affine and unsplit");
  // grouped: [E + 1] segment offsets and [E + 1] prefix sums of their 256-token tiles
  int *seg = reinterpret_cast<int *>(smem + S * C::STAGE_BYTES + 512 + C::EPI_BYTES);
  int *mtp = seg + kGroupMaxE + 2;
  if (GROUPED && threadIdx.x == 64) {  // warp 2 (otherwise idle) reads the segments
    int run = 0;
    for (int e = 0; e <= prm.E; ++e) {
      seg[e] = __ldg(prm.offsets + e);
      mtp[e] = run;
      if (e < prm.E) run += (__ldg(prm.offsets + e + 1) - seg[e] + 255) / 256;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&a_full[s], 8);  // one warp per TMEM lane quadrant, in each CTA
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * 4 * kDequantPerQuadrant);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before either uses the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = GROUPED ? prm.n_tiles * mtp[prm.E] : prm.m_tiles * prm.n_tiles;
  // Tile origin: first token m0, first W row n0 within the expert (grouped) or
  // the matrix, the expert's first row of the stacked W, and the end of the
  // tile's token rows.
  auto origin = [&](int tile, int &m0, int &n0, int64_t &wbase, int &mend) {
    if constexpr (GROUPED) {
      const int nt = tile % prm.n_tiles, mg = tile / prm.n_tiles;
      int lo = 0, hi = prm.E - 1;  // the segment e with mtp[e] <= mg < mtp[e + 1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mtp[mid] <= mg) lo = mid; else hi = mid - 1;
      }
      m0 = seg[lo] + (mg - mtp[lo]) * 256;
      n0 = nt * 256;
      wbase = static_cast<int64_t>(lo) * prm.N;
      mend = seg[lo + 1];
    } else {
      tile_origin(prm, tile, BN, 256, m0, n0);
      wbase = 0;
      mend = prm.M;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (each CTA)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&x_map)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&w_map)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      PairCursor<SPLIT> cur = GROUPED ? PairCursor<SPLIT>(prm, pair, npairs, KB, total_tiles) : PairCursor<SPLIT>(prm, pair, npairs, KB);
      PairItem item;
      while (ok && cur.next(item)) {
        int m0, n0, mend;
        int64_t wbase;
        origin(item.tile, m0, n0, wbase, mend);
        const int xrow = m0 + static_cast<int>(rank) * C::XH;
        const int wrow = static_cast<int>(wbase) + n0 + static_cast<int>(rank) * 128;
        for (int kb = item.kb0; kb < item.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          if (r >= 1 && !(ok = mbar_wait_cluster(&empty[s], (r - 1) & 1, abort_flag, kFaultProducerWait))) break;
          uint8_t *xs = smem + s * C::STAGE_BYTES;
          uint8_t *ws = xs + C::X_BYTES;
          mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::W_BYTES);
#pragma unroll
          for (int a = 0; a < C::BK / 64; ++a)
            tma_load_2d(xs + a * C::XH * 128, &x_map, &full[s], kb * C::BK + a * 64, xrow);
          tma_load_2d(ws, &w_map, &full[s], kb * C::BKW, wrow);
        }
      }
      const uint32_t issued = it;
      for (uint32_t j = (issued > static_cast<uint32_t>(S) ? issued - S : 0); j < issued; ++j)
        mbar_drain(&full[j % S], (j / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (CTA 0)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_pair(BN);
      uint32_t it = 0, t = 0;
      bool ok = true;
      PairCursor<SPLIT> cur = GROUPED ? PairCursor<SPLIT>(prm, pair, npairs, KB, total_tiles) : PairCursor<SPLIT>(prm, pair, npairs, KB);
      PairItem item;
      for (; ok && cur.next(item); ++t) {
        const int kb0 = item.kb0;
        if (t >= 1 && !(ok = mbar_wait_cluster(acc_empty, (t - 1) & 1, abort_flag, kFaultMmaWait))) break;
        tc_fence_after();
        for (int kb = kb0; kb < item.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          // a_full: both CTAs' A stages are written, and each dequant warp saw its CTA's stage land
          if (!(ok = mbar_wait_cluster(&a_full[s], r & 1, abort_flag, kFaultMmaWait))) break;
          tc_fence_after();
          const uint32_t xs_addr = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t a_tmem = tmem_base + C::A_COL0 + s * C::A_COLS;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint32_t b_addr = xs_addr + (kk / 4) * C::XH * 128 + (kk % 4) * 32;
            tc_mma_pair(tmem_base + kAccCol, a_tmem + kk * 8, sw128_kmajor_desc(b_addr), idesc,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(&empty[s]);
        }
        if (ok) tc_commit_pair(acc_full);
      }
      if (it > 0) mbar_drain(&empty[(it - 1) % S], ((it - 1) / S) & 1);
    }
  } else if (warp >= kDequantWarp0) {
    // ------------------------------------------------------------------ dequant + epilogue (each CTA)
    const int q = warp & 3;
    const int h = (warp - kDequantWarp0) >> 2;
    constexpr int H = kDequantPerQuadrant;
    const int row = q * 32 + lane;
    constexpr int CH = C::BK / 32;
    const int widx = warp - kDequantWarp0;
    uint8_t *ebox = smem + S * C::STAGE_BYTES + 512 + widx * 2048;  // this warp's output box
    uint32_t it0 = 0, t = 0;
    bool ok = true;
    PairCursor<SPLIT> cur = GROUPED ? PairCursor<SPLIT>(prm, pair, npairs, KB, total_tiles) : PairCursor<SPLIT>(prm, pair, npairs, KB);
    PairItem item;
    for (; ok && cur.next(item); ++t) {
      const int tile = item.tile, kb0 = item.kb0, kb1 = item.kb1;
      int m0, n0, mend;
      int64_t wbase;
      origin(tile, m0, n0, wbase, mend);
      const uint32_t itb = it0;  // ring position of this item's first K block
      it0 += static_cast<uint32_t>(kb1 - kb0);
      const int n = n0 + static_cast<int>(rank) * 128 + row;
      const bool row_ok = n < prm.N;
      const int64_t g_row = (wbase + (row_ok ? n : 0)) * prm.Gn;
      // Block-scaled formats: this row's power of two 2^-B (from its largest
      // scale byte; positive E4M3 and E8M0 order like their bits) keeps every
      // dequantized value within fp16; the epilogue multiplies by 2^B (nvfp4:
      // and by the tensor scale).
      const uint8_t *sbrow = nullptr;
      int bexp = 0;
      float rowfac = 1.0f;
      if constexpr (FMT != 0) {
        sbrow = prm.bscales + static_cast<int64_t>(row_ok ? n : 0) * prm.sb_row;
        const uint32_t mx = row_ok ? row_max_byte(sbrow, prm.sb_row) : 0u;
        if constexpr (FMT == 2) {
          const float vmax = e4m3_value(mx);
          bexp = vmax > 0.0f ? static_cast<int>((__float_as_uint(vmax) >> 23) & 0xFFu) - 127 + 1 - 13 : 0;
          rowfac = pow2f_exact(bexp) * __ldg(prm.gscale);
        } else {
          bexp = static_cast<int>(mx) - 127 - (FMT == 1 ? 13 : 7);
          rowfac = pow2f_exact(bexp);
        }
      }
      auto load_sb = [&](int kb, uint16_t (&sc)[CH], uint16_t (&bi)[CH]) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          if constexpr (FMT == 0) {
            const int g = (kb * C::BK + c * 32) / prm.G;
            const bool in = row_ok && kb < kb1 && g < prm.Gn;
            sc[c] = in ? ldg_nc2(prm.scales + g_row + g) : uint16_t(0);
            bi[c] = in ? ldg_nc2(prm.biases + g_row + g) : uint16_t(0);
          } else {
            const int g32 = (kb * C::BK + c * 32) / 32;  // the chunk's 32-code span
            const bool in = row_ok && kb < kb1 && g32 < prm.K / 32;
            sc[c] = !in ? uint16_t(0) : FMT == 2 ? ldg_nc2(sbrow + 2 * g32) : static_cast<uint16_t>(sbrow[g32]);
            bi[c] = 0;
          }
        }
      };
      // a queue of the next kSbAhead turns' scales, shifted by one each turn
      // (static indices keep it in registers)
      uint16_t sc_pf[kSbAhead][CH], bi_pf[kSbAhead][CH];
#pragma unroll
      for (int i = 0; i < kSbAhead; ++i) load_sb(kb0 + h + i * H, sc_pf[i], bi_pf[i]);
      for (int kb = kb0 + h; kb < kb1; kb += H) {
        const uint32_t it = itb + static_cast<uint32_t>(kb - kb0);
        const int s = it % S;
        const uint32_t r = it / S;
        uint16_t sc[CH], bi[CH];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          sc[c] = sc_pf[0][c];
          bi[c] = bi_pf[0][c];
        }
#pragma unroll
        for (int i = 0; i + 1 < kSbAhead; ++i)
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            sc_pf[i][c] = sc_pf[i + 1][c];
            bi_pf[i][c] = bi_pf[i + 1][c];
          }
        load_sb(kb + kSbAhead * H, sc_pf[kSbAhead - 1], bi_pf[kSbAhead - 1]);
        if (!(ok = mbar_wait(&full[s], r & 1, abort_flag, kFaultDequantWait))) break;
        if (r >= 1 && !(ok = mbar_wait_cluster(&empty[s], (r - 1) & 1, abort_flag, kFaultDequantWait))) break;
        __syncwarp();
        const uint32_t *wrow =
            reinterpret_cast<const uint32_t *>(smem + s * C::STAGE_BYTES + C::X_BYTES) + row * C::BKW;
        const uint32_t a_tmem = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::A_COL0 + s * C::A_COLS;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          uint32_t wv[BITS];
          if constexpr (BITS == 4) {
            const uint4 v4 = *reinterpret_cast<const uint4 *>(wrow + c * 4);
            wv[0] = v4.x; wv[1] = v4.y; wv[2] = v4.z; wv[3] = v4.w;
          } else if constexpr (BITS == 8) {
            const uint4 a4 = reinterpret_cast<const uint4 *>(wrow + c * 8)[0];
            const uint4 b4 = reinterpret_cast<const uint4 *>(wrow + c * 8)[1];
            wv[0] = a4.x; wv[1] = a4.y; wv[2] = a4.z; wv[3] = a4.w;
            wv[4] = b4.x; wv[5] = b4.y; wv[6] = b4.z; wv[7] = b4.w;
          } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) wv[i] = wrow[c * BITS + i];
          }
          uint32_t packed_cols[16];
          if constexpr (FMT == 0) {
            dequant_chunk_f16<BITS>(wv, sc[c], bi[c], packed_cols);
          } else if constexpr (FMT == 1) {
            const __half2 f = __float2half2_rn(pow2f_exact(static_cast<int>(sc[c]) - 127 - bexp));
            dequant_chunk_e2m1(reinterpret_cast<const uint32_t(&)[4]>(wv), f, f, packed_cols);
          } else if constexpr (FMT == 2) {
            const float p2 = pow2f_exact(-bexp);
            const __half2 f0 = __float2half2_rn(e4m3_value(sc[c] & 0xFFu) * p2);
            const __half2 f1 = __float2half2_rn(e4m3_value(sc[c] >> 8) * p2);
            dequant_chunk_e2m1(reinterpret_cast<const uint32_t(&)[4]>(wv), f0, f1, packed_cols);
          } else {
            const __half2 f = __float2half2_rn(pow2f_exact(static_cast<int>(sc[c]) - 127 - bexp + 8));
            dequant_chunk_e4m3(reinterpret_cast<const uint32_t(&)[8]>(wv), f, packed_cols);
          }
          tmem_st16(a_tmem + c * 16, packed_cols);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_at(&a_full[s], 0);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      if (!(ok = mbar_wait_cluster(acc_full, t & 1, abort_flag, kFaultEpilogueWait))) break;
      __syncwarp();
      tc_fence_after();
      const int bn0 = n0 + static_cast<int>(rank) * 128 + q * 32;
      // Row scale of token m0 + col + lane (the lane's token in a 32-column block).
      auto load_rs = [&](int col) {
        const int mlane = m0 + col + lane;
        return mlane < prm.M ? __ldg(prm.row_scale + mlane) : 0.0f;
      };
      // One 32-column block: this warp's 32 rows x 32 tokens (v, fp32 sums of
      // lane `lane`'s row), scaled and rounded into a shared-memory box
      // (token-major, the layout of y) and written by one TMA store, which
      // clips rows past N and tokens past M.
      auto emit_box = [&](int col, const float (&v)[32], float rs) {
        if (GROUPED && m0 + col + 32 > mend) {
          // the box crosses the end of the segment: plain stores of its rows in
          // the segment (the tokens past it belong to the next expert)
          if (m0 + col >= mend) return;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float rsi = __shfl_sync(0xffffffffu, rs, i);
            if (m0 + col + i < mend && bn0 + lane < prm.N)
              prm.y[static_cast<int64_t>(m0 + col + i) * prm.N + bn0 + lane] = __float2bfloat16_rn(v[i] * rsi);
          }
          return;
        }
        if (lane == 0) bulk_wait_read<0>();  // the store that last read this box is done with it
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float rsi = __shfl_sync(0xffffffffu, rs, i);
          const float out = FMT == 0 ? v[i] * rsi : v[i] * rsi * rowfac;  // (rowfac: this lane's W row)
          *reinterpret_cast<__nv_bfloat16 *>(ebox + i * 64 + lane * 2) = __float2bfloat16_rn(out);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the copy engine reads the box
        __syncwarp();
        if (lane == 0 && bn0 < prm.N && m0 + col < mend) {  // (a box wholly past the edges is not stored)
          tma_store_2d(&y_map, ebox, bn0, m0 + col);
          bulk_commit();
        }
      };
      if constexpr (!SPLIT) {
#pragma unroll 1
        for (int col = h * 32; col < BN; col += H * 32) {
          uint32_t v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kAccCol + col, v);
          const float rs = load_rs(col);  // (in flight with the accumulator read)
          tmem_ld_wait();
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          emit_box(col, f, rs);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_at(acc_empty, 0);
      } else {
        // This part's sums of the warp's blocks go to `partial`, which frees
        // the accumulator; the warp that arrives last on this (tile, CTA,
        // warp) counter adds every part's sums in part order, so the result
        // does not depend on which part finished last.  Layout: [part][tile]
        // [CTA][quadrant][32-token block] chunks of 32 rows x 32 tokens, each
        // as [token / 4][row][token % 4], so that one float4 store or load of
        // the warp covers 512 contiguous bytes.
        const int T = prm.m_tiles * prm.n_tiles;
        auto chunk = [&](int part, int col) {
          return reinterpret_cast<float4 *>(prm.partial) +
                 ((((static_cast<int64_t>(part) * T + tile) * 2 + rank) * 4 + q) * (BN / 32) + col / 32) * 256 + lane;
        };
#pragma unroll 1
        for (int col = h * 32; col < BN; col += H * 32) {
          uint32_t v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kAccCol + col, v);
          tmem_ld_wait();
          float4 *dst = chunk(item.part, col);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            __stcg(dst + i * 32, make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                             __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
        }
        tc_fence_before();
        __syncwarp();  // (also: every lane's partial sums are written)
        uint32_t before = 0;
        if (lane == 0) {
          mbar_arrive_at(acc_empty, 0);
          __threadfence();  // the warp's partial sums are visible before its count (a cumulative fence)
          before = atomicAdd(prm.arrivals + (tile * 2 + static_cast<int>(rank)) * (4 * H) + widx, 1u);
          // the last part: the other parts' counts seen here order their sums before the reads below
          if (before == static_cast<uint32_t>(prm.ksplit - 1)) __threadfence();
        }
        before = __shfl_sync(0xffffffffu, before, 0);
        __syncwarp();
        if (before == static_cast<uint32_t>(prm.ksplit - 1)) {
#pragma unroll 1
          for (int col = h * 32; col < BN; col += H * 32) {
            const float rs = load_rs(col);
            float v[32];
#pragma unroll 1
            for (int k = 0; k < prm.ksplit; ++k) {  // in part order
              const float4 *src = chunk(k, col);
              float4 f[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] = __ldcg(src + i * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                if (k == 0) {
                  v[4 * i] = f[i].x; v[4 * i + 1] = f[i].y; v[4 * i + 2] = f[i].z; v[4 * i + 3] = f[i].w;
                } else {
                  v[4 * i] += f[i].x; v[4 * i + 1] += f[i].y; v[4 * i + 2] += f[i].z; v[4 * i + 3] += f[i].w;
                }
              }
            }
            emit_box(col, v, rs);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // this warp's output stores have completed
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no MMA of the pair and no accumulator read is outstanding in either CTA
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Pre-pass: x bf16 [M, K] -> x16 fp16 [M, K] and row_scale[M], with
// x[m, k] = row_scale[m] * x16[m, k] exactly for every x16 that is a normal
// fp16 value.  row_scale[m] = 2^e with e = floor(log2(max_k |x[m, k]|)) - 14,
// so the row maximum of x16 lies in [2^14, 2^15) (far from fp16 overflow).
// One CTA per row; two vectorized passes over the row (the second hits L2).
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 256;

template <int BITS>
__global__ void __launch_bounds__(kPrepThreads) x_to_f16_rows_kernel(const __nv_bfloat16 *__restrict__ x, int K,
                                                                     __half *__restrict__ x16,
                                                                     float *__restrict__ row_scale,
                                                                     uint32_t *__restrict__ zero = nullptr,
                                                                     int nzero = 0) {
  __shared__ float red[kPrepThreads / 32];
  const int64_t m = blockIdx.x;
  if (m == 0)  // counters of the matmul that follows
    for (int i = threadIdx.x; i < nzero; i += kPrepThreads) zero[i] = 0;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + m * K);
  const int n16 = K / 16;  // 16-element steps (K is a multiple of 32)
  float amax = 0.0f;
  for (int i = threadIdx.x; i < 2 * n16; i += kPrepThreads) {
    const uint4 v = ldg_nc16(src + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      amax = fmaxf(amax, fabsf(__uint_as_float(u[hh] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(u[hh] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  // exponent of amax (bf16 keeps fp32's 8-bit exponent, so this is exact)
  int e = 0;
  if (amax > 0.0f) e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 14;
  // 2^-e and 2^e as exact fp32 powers of two (|e| <= 141 needs two factors)
  const float down_a = __uint_as_float(static_cast<uint32_t>(127 - e / 2) << 23);
  const float down_b = __uint_as_float(static_cast<uint32_t>(127 - (e - e / 2)) << 23);
  if (threadIdx.x == 0) {
    const float up_a = __uint_as_float(static_cast<uint32_t>(127 + e / 2) << 23);
    const float up_b = __uint_as_float(static_cast<uint32_t>(127 + (e - e / 2)) << 23);
    row_scale[m] = up_a * up_b;
  }
  uint4 *dst = reinterpret_cast<uint4 *>(x16 + m * K);
  for (int i = threadIdx.x; i < n16; i += kPrepThreads) {
    const uint4 v0 = ldg_nc16(src + 2 * i), v1 = ldg_nc16(src + 2 * i + 1);
    const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int e2 = 0; e2 < 16; ++e2)
      f[e2] = __uint_as_float(e2 & 1 ? (u[e2 >> 1] & 0xFFFF0000u) : (u[e2 >> 1] << 16)) * down_a * down_b;
    uint32_t o[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      constexpr int B = kx_block(BITS);
      const int e0 = (B == 16) ? kx_perm(BITS, 2 * t) : (B == 8 ? (2 * t >= 8 ? 8 : 0) + kx_perm(BITS, (2 * t) % 8) : 2 * t);
      const int e1 = (B == 16) ? kx_perm(BITS, 2 * t + 1)
                               : (B == 8 ? (2 * t + 1 >= 8 ? 8 : 0) + kx_perm(BITS, (2 * t + 1) % 8) : 2 * t + 1);
      __half2 p = __floats2half2_rn(f[e0], f[e1]);
      o[t] = *reinterpret_cast<uint32_t *>(&p);
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
inline int64_t round256(int64_t b) { return (b + 255) / 256 * 256; }

// The activations' workspace: x16 (fp16 [M, K]) + row_scale (fp32 [M]), each 256-byte padded.
inline size_t x16_bytes(int64_t M, int64_t K) { return static_cast<size_t>(round256(M * K * 2) + round256(M * 4)); }

// CTA-pair tiles (256 W rows x 256 tokens) of an M x N product.
inline int64_t pair_tiles(int64_t M, int64_t N) { return ((M + 255) / 256) * ((N + 255) / 256); }

// The pair kernel serves every M > 128 whose y rows are whole 16-byte units.
inline bool pick_shape_is_pair(int64_t M, int64_t N) { return M > 128 && N % 8 == 0; }

// K parts per tile of a pair launch.  When the tiles fill at most half of the
// 74 CTA pairs of a 148-SM part, each tile's K range is cut into up to four
// parts (one work item each, at least 32 K blocks per part), so that more
// pairs work; the parts' fp32 sums meet in the workspace.  (Sharing out only
// the last wave's tiles among all pairs, "stream-K", measured slower here: a
// shared tile costs its pairs ~4 us to publish their sums and the last one
// 6-8 us to add them, more than the idle pairs of a last wave cost.)  The
// choice depends on the shape alone, so the workspace size is known before
// the launch.
inline int pair_ksplit(int64_t M, int64_t N, int64_t K, int bits) {
  constexpr int64_t kPairs = 74;
  const int64_t T = pair_tiles(M, N);
  const int64_t KB = (K + (bits == 3 ? 127 : 63)) / (bits == 3 ? 128 : 64);
  const int64_t ks = std::min<int64_t>(std::min<int64_t>(kPairs / T, 4), KB / 32);
  return ks >= 2 ? static_cast<int>(ks) : 1;
}

// Workspace bytes of the split beyond the activations' part: one arrival
// counter per (tile, CTA, dequant warp), 256-byte padded, then [ksplit][tile]
// [CTA][128 rows][256 tokens] fp32 partial sums.
inline size_t pair_split_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  const int ks = pair_ksplit(M, N, K, bits);
  if (ks == 1) return 0;
  const int64_t T = pair_tiles(M, N);
  return static_cast<size_t>(round256(T * 2 * 4 * kDequantPerQuadrant * 4) + ks * T * 2 * 128 * 256 * 4);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int BITS, int BN>
cudaError_t launch_t(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                     const uint16_t *biases, int64_t N, int G, uint16_t *y, void *workspace, cudaStream_t stream) {
  using C = Cfg<BITS, BN>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  __half *x16 = reinterpret_cast<__half *>(workspace);
  float *row_scale = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + ((M * K * 2 + 255) / 256) * 256);
  x_to_f16_rows_kernel<BITS><<<static_cast<unsigned>(M), kPrepThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(x), static_cast<int>(K), x16, row_scale);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  CUtensorMap x_map, w_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(BN)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t P = K * BITS / 32;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(P) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::BKW), 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.offsets = nullptr;
  prm.E = 0;
  prm.bscales = nullptr;
  prm.sb_row = 0;
  prm.gscale = nullptr;
  prm.scales = reinterpret_cast<const __half *>(scales);
  prm.biases = reinterpret_cast<const __half *>(biases);
  prm.row_scale = row_scale;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = G;
  prm.Gn = static_cast<int>(K / G);
  prm.m_tiles = static_cast<int>((M + BN - 1) / BN);
  prm.n_tiles = static_cast<int>((N + 127) / 128);
  // Tile order: the CTAs in flight share either the x16 rows of all token
  // tiles (token tiles fastest: all of x16 stays hot in L2) or all of W (W-row
  // tiles fastest).  Keep hot whichever of the two is smaller.
  const int64_t w_bytes = N * K * BITS / 8 + 4 * N * (K / G);
  prm.n_fastest = (2 * M * K > w_bytes) ? 1 : 0;
#ifdef AQ_QMM_FORCE_ORDER  // build-time override (0: token tiles fastest, 1: W tiles fastest, else choose)
  if (AQ_QMM_FORCE_ORDER == 0 || AQ_QMM_FORCE_ORDER == 1) prm.n_fastest = AQ_QMM_FORCE_ORDER;
#endif

  auto kern = qmm_kernel<BITS, BN>;
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) != cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  const int64_t tiles = static_cast<int64_t>(prm.m_tiles) * prm.n_tiles;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(x_map, w_map, prm);
  return cudaGetLastError();
}

// Block-scaled prefill (FMT 1 mxfp4, 2 nvfp4, 3 mxfp8) on the single-CTA
// kernel: codes as the affine 4-bit / 8-bit layouts, one scale byte per 32
// (or 16) codes, and the dequantization of tc05.cuh.
template <int FMT, int BN>
cudaError_t launch_fmt_t(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint8_t *bscales,
                         const float *gscale, int64_t N, uint16_t *y, void *workspace, cudaStream_t stream) {
  constexpr int BITS = FMT == 3 ? 8 : 4;
  using C = Cfg<BITS, BN>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  __half *x16 = reinterpret_cast<__half *>(workspace);
  float *row_scale = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + ((M * K * 2 + 255) / 256) * 256);
  x_to_f16_rows_kernel<BITS><<<static_cast<unsigned>(M), kPrepThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(x), static_cast<int>(K), x16, row_scale);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  CUtensorMap x_map, w_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(BN)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t P = K * BITS / 32;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(P) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::BKW), 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.offsets = nullptr;
  prm.E = 0;
  prm.bscales = bscales;
  prm.sb_row = static_cast<int>(FMT == 2 ? K / 16 : K / 32);
  prm.gscale = gscale;
  prm.scales = nullptr;
  prm.biases = nullptr;
  prm.row_scale = row_scale;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = 32;
  prm.Gn = static_cast<int>(K / 32);
  prm.m_tiles = static_cast<int>((M + BN - 1) / BN);
  prm.n_tiles = static_cast<int>((N + 127) / 128);
  const int64_t w_bytes = N * K * BITS / 8 + prm.sb_row * N;
  prm.n_fastest = (2 * M * K > w_bytes) ? 1 : 0;
  auto kern = qmm_kernel<BITS, BN, FMT>;
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) != cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  const int64_t tiles = static_cast<int64_t>(prm.m_tiles) * prm.n_tiles;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(x_map, w_map, prm);
  return cudaGetLastError();
}

// Grouped launch: x [T, K] holds E segments of token rows (device offsets
// [E + 1]); segment e is multiplied by expert e of the stacked W [E*N, K], all
// in one persistent launch whose tile count each CTA reads from the offsets.
template <int BITS, int BN>
cudaError_t launch_grouped_t(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed, const uint16_t *scales,
                             const uint16_t *biases, int64_t E, int64_t N, int G, const int32_t *offsets, uint16_t *y,
                             void *workspace, cudaStream_t stream) {
  using C = Cfg<BITS, BN>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  __half *x16 = reinterpret_cast<__half *>(workspace);
  float *row_scale = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + ((T * K * 2 + 255) / 256) * 256);
  x_to_f16_rows_kernel<BITS><<<static_cast<unsigned>(T), kPrepThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(x), static_cast<int>(K), x16, row_scale);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  CUtensorMap x_map, w_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(BN)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t P = K * BITS / 32;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(E * N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(P) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::BKW), 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.offsets = offsets;
  prm.E = static_cast<int>(E);
  prm.bscales = nullptr;
  prm.sb_row = 0;
  prm.gscale = nullptr;
  prm.scales = reinterpret_cast<const __half *>(scales);
  prm.biases = reinterpret_cast<const __half *>(biases);
  prm.row_scale = row_scale;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(T);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = G;
  prm.Gn = static_cast<int>(K / G);
  prm.m_tiles = 0;  // from the offsets, on the device
  prm.n_tiles = static_cast<int>((N + 127) / 128);
  prm.n_fastest = 1;
  auto kern = qmm_kernel<BITS, BN>;
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) != cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  // at most ceil(T / BN) + E token tiles (each segment adds at most one partial tile)
  const int64_t bound = static_cast<int64_t>(prm.n_tiles) * ((T + BN - 1) / BN + E);
  const int grid = static_cast<int>(std::min<int64_t>(bound, sms));
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(x_map, w_map, prm);
  return cudaGetLastError();
}

// FMT 0: affine (scales, biases per G codes); 1 mxfp4, 2 nvfp4, 3 mxfp8: the
// block scales in bscales (rows of K/32 bytes, K/16 for nvfp4) and nvfp4's
// tensor scale in gscale (device memory).
template <int BITS, int BN, int FMT = 0>
cudaError_t launch_pair(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                        const uint16_t *biases, int64_t N, int G, uint16_t *y, void *workspace, size_t ws_bytes,
                        cudaStream_t stream, const uint8_t *bscales = nullptr, const float *gscale = nullptr) {
  using C = PairCfg<BITS, BN>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  __half *x16 = reinterpret_cast<__half *>(ws);
  float *row_scale = reinterpret_cast<float *>(ws + round256(M * K * 2));
  // the K split, when the caller's workspace holds its counters and partial sums
  static_assert(BN == 256, "the split's workspace is sized for 256-token tiles");
  int ksplit = pair_ksplit(M, N, K, BITS);
  const size_t base = x16_bytes(M, K);
  if (ksplit > 1 && ws_bytes < base + pair_split_bytes(M, N, K, BITS)) ksplit = 1;
  uint32_t *arrivals = ksplit > 1 ? reinterpret_cast<uint32_t *>(ws + base) : nullptr;
  const int n_arrivals = ksplit > 1 ? static_cast<int>(pair_tiles(M, N) * 2 * 4 * kDequantPerQuadrant) : 0;
  float *partial = ksplit > 1 ? reinterpret_cast<float *>(ws + base + round256(int64_t(n_arrivals) * 4)) : nullptr;
  x_to_f16_rows_kernel<BITS><<<static_cast<unsigned>(M), kPrepThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(x), static_cast<int>(K), x16, row_scale, arrivals, n_arrivals);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  CUtensorMap x_map, w_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(C::XH)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t P = K * BITS / 32;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(P) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::BKW), 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap y_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&y_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.offsets = nullptr;
  prm.E = 0;
  prm.bscales = FMT == 0 ? nullptr : bscales;
  prm.sb_row = FMT == 0 ? 0 : static_cast<int>(FMT == 2 ? K / 16 : K / 32);
  prm.gscale = FMT == 0 ? nullptr : gscale;
  prm.scales = reinterpret_cast<const __half *>(scales);
  prm.biases = reinterpret_cast<const __half *>(biases);
  prm.row_scale = row_scale;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = FMT == 0 ? G : 32;
  prm.Gn = static_cast<int>(K / prm.G);
  prm.m_tiles = static_cast<int>((M + BN - 1) / BN);
  prm.n_tiles = static_cast<int>((N + 255) / 256);
  const int64_t w_bytes = N * K * BITS / 8 + (FMT == 0 ? 4 * N * (K / G) : static_cast<int64_t>(prm.sb_row) * N);
  prm.n_fastest = (2 * M * K > w_bytes) ? 1 : 0;
#ifdef AQ_QMM_FORCE_ORDER
  if (AQ_QMM_FORCE_ORDER == 0 || AQ_QMM_FORCE_ORDER == 1) prm.n_fastest = AQ_QMM_FORCE_ORDER;
#endif
  prm.ksplit = ksplit;
  prm.partial = partial;
  prm.arrivals = arrivals;

  auto kern = ksplit > 1 ? qmm_pair_kernel<BITS, BN, true, FMT> : qmm_pair_kernel<BITS, BN, false, FMT>;
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    for (auto k : {qmm_pair_kernel<BITS, BN, true, FMT>, qmm_pair_kernel<BITS, BN, false, FMT>})
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  const int64_t items = static_cast<int64_t>(prm.m_tiles) * prm.n_tiles * ksplit;
  const int pairs = static_cast<int>(std::min<int64_t>(items, std::max(1, sms / 2)));
  kern<<<2 * pairs, kThreads, C::SMEM_BYTES, stream>>>(x_map, w_map, y_map, prm);
  return cudaGetLastError();
}

// Grouped launch on CTA pairs (see launch_grouped_t): token tiles of 256 rows
// per segment, W tiles of 256 rows of the segment's expert.
template <int BITS>
cudaError_t launch_pair_grouped(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed,
                                const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G,
                                const int32_t *offsets, uint16_t *y, void *workspace, cudaStream_t stream) {
  using C = PairCfg<BITS, 256>;
  constexpr size_t kSmem = C::SMEM_BYTES + kGroupTabBytes;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  __half *x16 = reinterpret_cast<__half *>(ws);
  float *row_scale = reinterpret_cast<float *>(ws + round256(T * K * 2));
  x_to_f16_rows_kernel<BITS><<<static_cast<unsigned>(T), kPrepThreads, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(x), static_cast<int>(K), x16, row_scale);
  cudaError_t pe = cudaGetLastError();
  if (pe != cudaSuccess) return pe;
  CUtensorMap x_map, w_map, y_map;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(C::XH)};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x16, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t P = K * BITS / 32;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(P), static_cast<cuuint64_t>(E * N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(P) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(C::BKW), 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&y_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Params prm;
  prm.offsets = offsets;
  prm.E = static_cast<int>(E);
  prm.bscales = nullptr;
  prm.sb_row = 0;
  prm.gscale = nullptr;
  prm.scales = reinterpret_cast<const __half *>(scales);
  prm.biases = reinterpret_cast<const __half *>(biases);
  prm.row_scale = row_scale;
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(T);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = G;
  prm.Gn = static_cast<int>(K / G);
  prm.m_tiles = 0;  // from the offsets, on the device
  prm.n_tiles = static_cast<int>((N + 255) / 256);
  prm.n_fastest = 1;
  prm.ksplit = 1;
  auto kern = qmm_pair_kernel<BITS, 256, false, 0, true>;
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem))) !=
        cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  // at most ceil(T / 256) + E token tiles (each segment adds at most one partial tile)
  const int64_t bound = static_cast<int64_t>(prm.n_tiles) * ((T + 255) / 256 + E);
  const int pairs = static_cast<int>(std::min<int64_t>(bound, std::max(1, sms / 2)));
  kern<<<2 * pairs, kThreads, kSmem, stream>>>(x_map, w_map, y_map, prm);
  return cudaGetLastError();
}

// Tile shape.  Measured on B200 (4-bit, G = 64, TFLOP/s, pair / one CTA at
// 256 / one CTA at 128 tokens): M = 512, 2048, 8192 at K = 4096, N = 14336:
// 532/540/344, 742/744/461, 901/895/510; at K = 14336, N = 4096: 501/383/485,
// 1016/763/571, 1197/946/611.  The CTA pair carries the most multiply-adds per
// staged byte and is never slower, so every M > 128 takes it.  Smaller M: one
// CTA per tile, the width that best trades wave fill against bytes moved per
// multiply-add (the x16 slice, BN x BK fp16, plus the packed W slice).
enum Shape { kPair256 = 0, kOne256 = 1, kOne128 = 2, kOne64 = 3 };

template <int BITS>
int pick_shape(int64_t M, int64_t N, int sms) {
#ifdef AQ_QMM_FORCE_SHAPE  // build-time override (0..3 as in Shape; else choose)
  if (AQ_QMM_FORCE_SHAPE >= 0 && AQ_QMM_FORCE_SHAPE <= 3) return AQ_QMM_FORCE_SHAPE;
#endif
  if (pick_shape_is_pair(M, N)) return kPair256;  // (the pair's output stores need 16-byte rows of y)
  auto score = [&](int64_t bn, int64_t bytes) {
    const int64_t t = ((M + bn - 1) / bn) * ((N + 127) / 128);
    const int64_t waves = (t + sms - 1) / sms;
    const double fill = static_cast<double>(t) / static_cast<double>(waves * sms);
    return fill * static_cast<double>(bn) / static_cast<double>(bytes);
  };
  const double s256 = score(256, Cfg<BITS, 256>::X_BYTES + Cfg<BITS, 256>::W_BYTES);
  const double s128 = score(128, Cfg<BITS, 128>::X_BYTES + Cfg<BITS, 128>::W_BYTES);
  const double s64 = score(64, Cfg<BITS, 64>::X_BYTES + Cfg<BITS, 64>::W_BYTES);
  if (M > 128 && s256 >= s128 && s256 >= s64) return kOne256;
  if (M > 64 && s128 >= s64) return kOne128;
  return kOne64;
}

template <int BITS>
cudaError_t launch_bits(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                        const uint16_t *biases, int64_t N, int G, uint16_t *y, void *ws, size_t ws_bytes,
                        cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 148;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  switch (pick_shape<BITS>(M, N, sms)) {
    case kPair256: return launch_pair<BITS, 256>(x, M, K, packed, scales, biases, N, G, y, ws, ws_bytes, s);
    case kOne256: return launch_t<BITS, 256>(x, M, K, packed, scales, biases, N, G, y, ws, s);
    case kOne128: return launch_t<BITS, 128>(x, M, K, packed, scales, biases, N, G, y, ws, s);
    default: return launch_t<BITS, 64>(x, M, K, packed, scales, biases, N, G, y, ws, s);
  }
}

}  // namespace qmm

// Block-scaled prefill: fmt 1 mxfp4, 2 nvfp4 (gscale: its tensor scale on the
// device), 3 mxfp8; token tile 64 / 128 / 256 by M as the affine single CTA.
cudaError_t launch_qmm_block_scaled(int fmt, const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed,
                                    const uint8_t *scales, const float *gscale, int64_t N, uint16_t *y, void *ws,
                                    size_t ws_bytes, cudaStream_t s) {
  // M > 128 (and N % 8 == 0): the CTA pair, as for the affine format
  if (qmm::pick_shape_is_pair(M, N)) {
    switch (fmt) {
      case 1: return qmm::launch_pair<4, 256, 1>(x, M, K, packed, nullptr, nullptr, N, 32, y, ws, ws_bytes, s, scales, gscale);
      case 2: return qmm::launch_pair<4, 256, 2>(x, M, K, packed, nullptr, nullptr, N, 16, y, ws, ws_bytes, s, scales, gscale);
      case 3: return qmm::launch_pair<8, 256, 3>(x, M, K, packed, nullptr, nullptr, N, 32, y, ws, ws_bytes, s, scales, gscale);
      default: return cudaErrorInvalidValue;
    }
  }
  const int bn = M <= 64 ? 64 : M <= 128 ? 128 : 256;
#define AQ_FMT_BN(F)                                                                                               \
  switch (bn) {                                                                                                    \
    case 64: return qmm::launch_fmt_t<F, 64>(x, M, K, packed, scales, gscale, N, y, ws, s);                       \
    case 128: return qmm::launch_fmt_t<F, 128>(x, M, K, packed, scales, gscale, N, y, ws, s);                     \
    default: return qmm::launch_fmt_t<F, 256>(x, M, K, packed, scales, gscale, N, y, ws, s);                      \
  }
  switch (fmt) {
    case 1: AQ_FMT_BN(1)
    case 2: AQ_FMT_BN(2)
    case 3: AQ_FMT_BN(3)
    default: return cudaErrorInvalidValue;
  }
#undef AQ_FMT_BN
}

// Grouped prefill (see launch_grouped_t): BN by the mean segment length.
cudaError_t launch_qmm_grouped(const uint16_t *x, int64_t T, int64_t K, const uint32_t *packed,
                               const uint16_t *scales, const uint16_t *biases, int64_t E, int64_t N, int G, int bits,
                               const int32_t *offsets, uint16_t *y, void *ws, cudaStream_t s) {
  if (E < 1 || E > qmm::kGroupMaxE) return cudaErrorInvalidValue;
  const int64_t mean = (T + E - 1) / E;
  // segments of more than 192 rows on average: CTA pairs (y rows of whole 16-byte units for the output stores)
  if (mean > 192 && N % 8 == 0) {
    switch (bits) {
      case 2: return qmm::launch_pair_grouped<2>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);
      case 3: return qmm::launch_pair_grouped<3>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);
      case 4: return qmm::launch_pair_grouped<4>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);
      default: return qmm::launch_pair_grouped<8>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);
    }
  }
  const int bn = mean <= 96 ? 64 : mean <= 384 ? 128 : 256;
#define AQ_GROUPED(B, N_)                                                                                          \
  case N_: return qmm::launch_grouped_t<B, N_>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);
#define AQ_GROUPED_BITS(B)                                                                                         \
  switch (bn) {                                                                                                    \
    AQ_GROUPED(B, 64)                                                                                              \
    AQ_GROUPED(B, 128)                                                                                             \
    default: return qmm::launch_grouped_t<B, 256>(x, T, K, packed, scales, biases, E, N, G, offsets, y, ws, s);    \
  }
  switch (bits) {
    case 2: AQ_GROUPED_BITS(2)
    case 3: AQ_GROUPED_BITS(3)
    case 4: AQ_GROUPED_BITS(4)
    default: AQ_GROUPED_BITS(8)
  }
#undef AQ_GROUPED_BITS
#undef AQ_GROUPED
}

bool qmm_supports(int64_t M, int64_t N, int64_t K, int G, int bits) {
  (void)G;
  if (M <= 0 || N <= 0 || K <= 0) return false;
  // TMA: the packed row pitch must be a multiple of 16 bytes.
  if ((K * bits) % 128 != 0) return false;
  return true;
}

// Workspace of the QMM paths' activations: x16 (fp16 [M, K]) + row_scale (fp32 [M]).
size_t qmm_workspace_bytes(int64_t M, int64_t K) { return qmm::x16_bytes(M, K); }

// Workspace of the affine QMM path: the activations' part plus, for a
// K-split CTA-pair launch, its counters and fp32 partial sums.
size_t qmm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  return qmm_workspace_bytes(M, K) + (qmm::pick_shape_is_pair(M, N) ? qmm::pair_split_bytes(M, N, K, bits) : 0);
}

// ws_bytes: the workspace's size; the K split runs only when it holds that part too.
cudaError_t launch_qmm(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, void *ws, size_t ws_bytes,
                       cudaStream_t s) {
  switch (bits) {
    case 2: return qmm::launch_bits<2>(x, M, K, packed, scales, biases, N, G, y, ws, ws_bytes, s);
    case 3: return qmm::launch_bits<3>(x, M, K, packed, scales, biases, N, G, y, ws, ws_bytes, s);
    case 4: return qmm::launch_bits<4>(x, M, K, packed, scales, biases, N, G, y, ws, ws_bytes, s);
    default: return qmm::launch_bits<8>(x, M, K, packed, scales, biases, N, G, y, ws, ws_bytes, s);
  }
}

cudaError_t read_and_clear_fault(uint32_t *word) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyFromSymbol(word, g_fault_word, sizeof(uint32_t))) != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_fault_word, &zero, sizeof(uint32_t));
}

}  // namespace aq
