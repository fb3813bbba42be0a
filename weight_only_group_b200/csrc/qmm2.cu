// QMM for prefill without any workspace: quantized matrix x matrix on the
// 5th-generation tensor cores (tcgen05 + tensor memory), sm_100a.
//
// Method: metalworking "MLX Quantization", section "Mechanics" (QMM is the
// prefill/batch case: dequantize weight tiles on chip, then a tiled GEMM
// against them; "One trap for intuition": dequantize on every use) and anllm
// "Tutorial 10: Quantization", section 5 (the fused product equals
// dequantize-then-multiply).
//
// Precision (as the workspace kernel in qmm.cu): both MMA operands are fp16.
// Weights are fp16_rn(fp32_rn(q*scale + bias)); each token row m of x is
// carried as fp16 x16 = x * 2^-e_m, e_m = floor(log2 max_k |x[m,k]|) - 14
// (an exact power-of-two scaling, so the row maximum of x16 lies in
// [2^14, 2^15)); the epilogue multiplies the fp32 accumulator by 2^e_m.
//
// No workspace.  A small pre-kernel computes e_m and parks it, as one byte per
// token row, inside the output y itself: in the region of every output tile
// that covers that row, at bytes that only that tile's epilogue overwrites.
// Each tile is computed by exactly one CTA, which reads its tile's bytes before
// its own epilogue writes the tile, so no CTA ever reads a byte another CTA
// writes.  The matmul kernel is launched as a programmatic dependent of the
// pre-kernel: its prologue and its weight loads overlap the pre-kernel.
//
// B200 design ("swap AB": weights are the MMA's A operand, tokens its N):
//  * CTA tile: 256 rows of W (two MMA blocks of M = 128: TMEM lanes are the W
//    rows, the two blocks use different TMEM columns) x 128 tokens (MMA
//    N = 128).  The two MMAs of a K slice share the x tile, so each x byte
//    brought into the SM feeds 256 W rows (the workspace kernel: 128).
//    Persistent CTAs walk the tiles, W-row tiles fastest, so concurrently
//    running CTAs share the x rows.
//  * Warp 0 (one lane): TMA producer: per K block the x tile [128 tokens x BK]
//    as raw bf16 (128-byte swizzle, the canonical K-major UMMA layout) and the
//    packed W tile [256 rows x BK*bits/32 words] into a ring of stages.
//  * Warps 2-3: convert the landed x tile in place, bf16 -> fp16 x * 2^-e_m,
//    in the K order the dequantized weights use, then make the writes visible
//    to the tensor core (fence.proxy.async).
//  * Warps 4..15 (three per TMEM lane quadrant): dequantize.  Thread (quadrant,
//    lane) owns W rows 32*quadrant + lane of both blocks; the quadrant's warps
//    take K blocks in turn and write the fp16 weights with tcgen05.st straight
//    into a TMEM stage, which the MMA reads as operand A.  The same warps run
//    the epilogue (tcgen05.ld, x 2^e_m, bf16 RNE store).
//  * Warp 1 (one lane): issues tcgen05.mma.kind::f16 (two per K slice) and
//    tcgen05.commit; warp 1 also owns the TMEM allocation.
//  * Every mbarrier wait is bounded; on expiry the kernel records a bit in its
//    fault word, stops issuing work and exits cleanly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "tc05.cuh"

namespace aq {

__device__ uint32_t g_qmm2_fault = 0;

namespace qmm {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();  // driver entry point, resolved once (qmm.cu)

namespace v2 {

constexpr int kBN = 128;         // tokens per CTA tile (the MMA's N)
constexpr int kConvWarp0 = 2;    // warps 2, 3 convert x
constexpr int kConvWarps = 2;
constexpr int kDeqWarp0 = 4;     // warps 4.. dequantize + epilogue
constexpr int kDeqPerQuad = 2;  // a divisor of every ring depth below (each warp owns fixed ring slots)
constexpr int kThreads = 32 * (kDeqWarp0 + 4 * kDeqPerQuad);
constexpr int kTmemCols = 512;

// WB: 128-row W blocks per CTA tile (two MMAs of M = 128 per K slice when 2).
template <int BITS, int WB>
struct Cfg {
  static constexpr int WROWS = 128 * WB;                     // W rows per CTA tile
  static constexpr int BK = (BITS == 3) ? 128 : 64;          // K per stage (elements)
  static constexpr int BKW = BK * BITS / 32;                 // packed words per W row per stage
  static constexpr int X_BYTES = kBN * BK * 2;               // x tile bytes (bf16 in, fp16 after conversion)
  static constexpr int W_BYTES = WROWS * BKW * 4;            // packed W tile bytes
  static constexpr int STAGE_BYTES = ((X_BYTES + W_BYTES + 1023) / 1024) * 1024;
  static constexpr int A_COLS = BK / 2;                      // TMEM columns of one 128-row A block
  static constexpr int ACC_COLS = WB * kBN;                  // accumulators: block b at column b * kBN
  static constexpr int TMEM_STAGES = (kTmemCols - ACC_COLS) / (WB * A_COLS);
  static constexpr int SMEM_BUDGET = 220 * 1024;
  // the ring depth: a multiple of the dequant warps per quadrant (2), so that
  // the iterations one warp takes always fall in the same ring slots
  static constexpr int STAGES = std::min(std::min(TMEM_STAGES, 8), SMEM_BUDGET / STAGE_BYTES) / 2 * 2;
  // at least half the SM's shared memory, so that no second CTA of this kernel
  // shares an SM (each CTA allocates all 512 TMEM columns)
  static constexpr int SMEM_BYTES =
      std::max(STAGES * STAGE_BYTES + 1024 /*align*/ + 4096 /*barriers, exponent tables*/, 116 * 1024);
  static_assert(STAGES >= 2 && STAGES % kDeqPerQuad == 0, "ring depth");
};

// Bounded wait on this kernel's fault word.
AQ_DEVICE bool wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t fault_bit) {
  return aq::mbar_wait(bar, parity, abort_flag, &g_qmm2_fault, fault_bit);
}

AQ_DEVICE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Byte offset, inside y, of the exponent byte of token i (0..127) of the tile
// whose first token is m0 and first W row n0 (tile width w = min(wrows, N - n0)
// columns): the tile region's rows are 2w bytes wide, filled in order.
__host__ __device__ inline int64_t exp_byte(int64_t m0, int64_t n0, int i, int64_t N, int wrows) {
  const int64_t w2 = 2 * std::min<int64_t>(wrows, N - n0);
  return (m0 + i / w2) * 2 * N + 2 * n0 + i % w2;
}

struct Params {
  const __nv_bfloat16 *x;
  const __half *scales, *biases;
  __nv_bfloat16 *y;
  int M, N, K, G, Gn;
  int m_tiles, n_tiles;
};

// ---------------------------------------------------------------------------
// Pre-kernel: one warp per token row m.  b = 0 for an all-zero row (e = 0),
// else 1 + the fp32 exponent field of max |x[m, :]| (e = b - 1 - 141, which is
// floor(log2 max) - 14 for a normal maximum and -141 for a subnormal one).
// The byte goes to every output tile that covers row m.
// ---------------------------------------------------------------------------
constexpr int kExpThreads = 256;

__global__ void __launch_bounds__(kExpThreads) qmm2_exponents_kernel(const __nv_bfloat16 *__restrict__ x, int M,
                                                                      int K, int N, int n_tiles, int wrows,
                                                                      uint8_t *__restrict__ y_bytes) {
  // the matmul launched after this kernel may start its prologue now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * (kExpThreads / 32) + (threadIdx.x >> 5);
  if (m >= M) return;
  const uint4 *row = reinterpret_cast<const uint4 *>(x + m * K);
  uint32_t mx = 0;  // largest |x| as bf16 magnitude bits (integer order = value order)
  for (int i = lane; i < K / 8; i += 32) {
    const uint4 v = ldg_nc16(row + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) mx = max(mx, max(u[j] & 0x7FFFu, (u[j] >> 16) & 0x7FFFu));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const uint8_t b = mx == 0 ? uint8_t(0) : static_cast<uint8_t>(((mx >> 7) & 0xFFu) + 1u);
  const int64_t m0 = m / kBN * kBN;
  const int i = static_cast<int>(m - m0);
  for (int nt = lane; nt < n_tiles; nt += 32) y_bytes[exp_byte(m0, static_cast<int64_t>(nt) * wrows, i, N, wrows)] = b;
}

// ---------------------------------------------------------------------------
// Conversion of one 16-byte chunk (8 bf16 of one token row) into fp16 x * 2^-e
// ---------------------------------------------------------------------------
// fp16x2 of (lo * f, hi * f) with f = fa * fb (two exact power-of-two factors).
AQ_DEVICE uint32_t to_f16x2(float lo, float hi, float fa, float fb) {
  const float2 v = __fmul2_rn(__fmul2_rn(make_float2(lo, hi), make_float2(fa, fa)), make_float2(fb, fb));
  const __half2 h = __floats2half2_rn(v.x, v.y);
  return *reinterpret_cast<const uint32_t *>(&h);
}
AQ_DEVICE float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
AQ_DEVICE float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int BITS, int WB>
__global__ void __launch_bounds__(kThreads, 1) qmm2_kernel(const __grid_constant__ CUtensorMap x_map,
                                                           const __grid_constant__ CUtensorMap w_map, Params prm) {
  using C = Cfg<BITS, WB>;
  constexpr int kWRows = C::WROWS;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);  // TMA landed x + W
  uint64_t *x_ready = full + S;     // converters done with the stage's x tile
  uint64_t *a_full = x_ready + S;   // dequantized A written to TMEM
  uint64_t *empty = a_full + S;     // MMAs of the stage completed (smem and TMEM stage free)
  uint64_t *acc_full = empty + S;
  uint64_t *acc_empty = acc_full + 1;
  uint64_t *exp_ready = acc_empty + 1;  // [2]: exponent table of a tile written
  uint64_t *exp_free = exp_ready + 2;   // [2]: the epilogue that used a table is done with it
  float *up = reinterpret_cast<float *>(exp_free + 2);    // [2][kBN]: 2^e of the tile's tokens
  float2 *down = reinterpret_cast<float2 *>(up + 2 * kBN);  // [2][kBN]: 2^-e as two factors
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(down + 2 * kBN);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_tiles = prm.m_tiles * prm.n_tiles;
  const int KB = (prm.K + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&x_ready[s], kConvWarps);
      mbar_init(&a_full[s], 4);  // one warp per TMEM lane quadrant fills a K block
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4 * kDeqPerQuad);
    mbar_init(&exp_ready[0], kConvWarps);
    mbar_init(&exp_ready[1], kConvWarps);
    mbar_init(&exp_free[0], 4 * kDeqPerQuad);
    mbar_init(&exp_free[1], 4 * kDeqPerQuad);
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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // x is complete before this grid starts (the pre-kernel, which it depends
    // on, only started after the work before it); W is never written.
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&x_map)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&w_map)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int n0 = (tile % prm.n_tiles) * kWRows;
        const int m0 = (tile / prm.n_tiles) * kBN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          if (r >= 1 && !(ok = wait(&empty[s], (r - 1) & 1, abort_flag, kFaultProducerWait))) break;
          uint8_t *xs = smem + s * C::STAGE_BYTES;
          uint8_t *ws = xs + C::X_BYTES;
          mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::W_BYTES);
#pragma unroll
          for (int a = 0; a < C::BK / 64; ++a) tma_load_2d(xs + a * kBN * 128, &x_map, &full[s], kb * C::BK + a * 64, m0);
          tma_load_2d(ws, &w_map, &full[s], kb * C::BKW, n0);
        }
      }
      const uint32_t issued = it;  // drain: every issued load must land before the CTA exits
      for (uint32_t j = (issued > static_cast<uint32_t>(S) ? issued - S : 0); j < issued; ++j)
        mbar_drain(&full[j % S], (j / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kBN);
      uint32_t it = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t) {
        if (t >= 1 && !(ok = wait(acc_empty, (t - 1) & 1, abort_flag, kFaultMmaWait))) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t r = it / S;
          if (!(ok = wait(&x_ready[s], r & 1, abort_flag, kFaultMmaWait))) break;
          if (!(ok = wait(&a_full[s], r & 1, abort_flag, kFaultMmaWait))) break;
          tc_fence_after();
          const uint32_t xs_addr = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t a_tmem = tmem_base + C::ACC_COLS + s * WB * C::A_COLS;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            // K = 16 slice kk: 32 bytes into a 128-byte swizzle row; a new atom column every 64 elements
            const uint64_t bd = sw128_kmajor_desc(xs_addr + (kk / 4) * kBN * 128 + (kk % 4) * 32);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
#pragma unroll
            for (int b = 0; b < WB; ++b) tc_mma_ts(tmem_base + b * kBN, a_tmem + b * C::A_COLS + kk * 8, bd, idesc, acc);
          }
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(acc_full);
      }
      if (it > 0) mbar_drain(&empty[(it - 1) % S], ((it - 1) / S) & 1);  // last MMAs done before TMEM is freed
    }
  } else if (warp < kDeqWarp0) {
    // ------------------------------------------------------------------ x converters
    const int ct = threadIdx.x - 32 * kConvWarp0;  // 0..63
    constexpr int NT = 32 * kConvWarps;
    uint32_t it = 0, t = 0;
    bool ok = true;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the exponent bytes are the pre-kernel's
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t) {
      const int64_t n0 = static_cast<int64_t>(tile % prm.n_tiles) * kWRows;
      const int64_t m0 = static_cast<int64_t>(tile / prm.n_tiles) * kBN;
      const int buf = t & 1;
      // the tile's exponent bytes (this CTA's epilogue of this tile overwrites
      // them later).  Each converter warp builds the whole table (both write the
      // same values), so no barrier between the two warps is needed.
      const uint8_t *yb = reinterpret_cast<const uint8_t *>(prm.y);
      uint8_t eb[kBN / 32];
#pragma unroll
      for (int j = 0; j < kBN / 32; ++j) {
        const int i = lane + 32 * j;
        eb[j] = (m0 + i < prm.M) ? yb[exp_byte(m0, n0, i, prm.N, kWRows)] : uint8_t(0);
      }
      // exponent table buf: free once the epilogue of tile t - 2 has used it
      if (t >= 2 && !(ok = wait(&exp_free[buf], ((t >> 1) - 1) & 1, abort_flag, kFaultDequantWait))) break;
#pragma unroll
      for (int j = 0; j < kBN / 32; ++j) {
        const int i = lane + 32 * j;
        const int e = eb[j] == 0 ? 0 : static_cast<int>(eb[j]) - 1 - 141;
        const int ea = e / 2, ebb = e - e / 2;
        up[buf * kBN + i] = __uint_as_float(static_cast<uint32_t>(127 + ea) << 23) *
                            __uint_as_float(static_cast<uint32_t>(127 + ebb) << 23);
        down[buf * kBN + i] = make_float2(__uint_as_float(static_cast<uint32_t>(127 - ea) << 23),
                                          __uint_as_float(static_cast<uint32_t>(127 - ebb) << 23));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&exp_ready[buf]);
      const float2 *dn = down + buf * kBN;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % S;
        const uint32_t r = it / S;
        if (!(ok = wait(&full[s], r & 1, abort_flag, kFaultDequantWait))) break;
        uint8_t *xs = smem + s * C::STAGE_BYTES;
        if constexpr (BITS == 2) {
          // K blocks of 16 (logical 16-byte chunks 2c, 2c+1 of a row): slot t
          // holds element (t % 2) * 8 + t / 2
          for (int item = ct; item < kBN * 4; item += NT) {
            const int row = item >> 2, cp = item & 3;
            const float2 f = dn[row];
            uint8_t *rp = xs + row * 128;
            uint4 *p0 = reinterpret_cast<uint4 *>(rp + (((2 * cp) ^ (row & 7)) << 4));
            uint4 *p1 = reinterpret_cast<uint4 *>(rp + (((2 * cp + 1) ^ (row & 7)) << 4));
            const uint4 a = *p0, b = *p1;
            const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // elements 2i, 2i+1 in u[i]
            auto el = [&](int k) { return (k & 1) ? bf_hi(u[k >> 1]) : bf_lo(u[k >> 1]); };
            uint32_t o[8];
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) o[tt] = to_f16x2(el(tt), el(tt + 8), f.x, f.y);
            *p0 = make_uint4(o[0], o[1], o[2], o[3]);
            *p1 = make_uint4(o[4], o[5], o[6], o[7]);
          }
        } else {
          constexpr int CHUNKS = C::X_BYTES / 16;
          for (int c = ct; c < CHUNKS; c += NT) {
            const int row = (c >> 3) % kBN;  // 8 chunks per 128-byte row; BK = 128 has two row blocks
            const float2 f = dn[row];
            uint4 *p = reinterpret_cast<uint4 *>(xs + c * 16);
            const uint4 a = *p;
            uint4 o;
            if constexpr (BITS == 4) {
              // K blocks of 8: slots hold elements 0,4,1,5,2,6,3,7
              o.x = to_f16x2(bf_lo(a.x), bf_lo(a.z), f.x, f.y);
              o.y = to_f16x2(bf_hi(a.x), bf_hi(a.z), f.x, f.y);
              o.z = to_f16x2(bf_lo(a.y), bf_lo(a.w), f.x, f.y);
              o.w = to_f16x2(bf_hi(a.y), bf_hi(a.w), f.x, f.y);
            } else {  // natural order
              o.x = to_f16x2(bf_lo(a.x), bf_hi(a.x), f.x, f.y);
              o.y = to_f16x2(bf_lo(a.y), bf_hi(a.y), f.x, f.y);
              o.z = to_f16x2(bf_lo(a.z), bf_hi(a.z), f.x, f.y);
              o.w = to_f16x2(bf_lo(a.w), bf_hi(a.w), f.x, f.y);
            }
            *p = o;
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core's reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_ready[s]);
      }
    }
  } else {
    // ------------------------------------------------------------------ dequant + epilogue
    const int q = warp & 3;                  // TMEM lane quadrant
    const int h = (warp - kDeqWarp0) >> 2;   // the quadrant's warps take iterations in turn: warp h
                                             // takes every global iteration it with it % H == h, so it
                                             // alone serves ring slots s with s % H == h (H divides S)
    constexpr int H = kDeqPerQuad;
    const int lrow = q * 32 + lane;          // row within a 128-row block == TMEM lane
    static_assert(WB == 1 || WB == 2, "one or two W blocks");
    constexpr int CH = C::BK / 32;           // 32-code chunks per row per K block
    asm volatile("griddepcontrol.wait;" ::: "memory");  // y holds the pre-kernel's bytes until the epilogue
    uint32_t it0 = 0, t = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++t, it0 += KB) {
      const int n0 = (tile % prm.n_tiles) * kWRows;
      const int m0 = (tile / prm.n_tiles) * kBN;
      const int nr[2] = {n0 + lrow, n0 + 128 + lrow};
      const bool rok[2] = {nr[0] < prm.N, WB == 2 && nr[1] < prm.N};
      const int64_t grow[2] = {static_cast<int64_t>(rok[0] ? nr[0] : 0) * prm.Gn,
                               static_cast<int64_t>(rok[1] ? nr[1] : 0) * prm.Gn};
      auto load_sb = [&](int kb, uint16_t (&sc)[2][CH], uint16_t (&bi)[2][CH]) {
#pragma unroll
        for (int b = 0; b < WB; ++b)
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const int g = (kb * C::BK + c * 32) / prm.G;
            const bool in = rok[b] && kb < KB && g < prm.Gn;
            sc[b][c] = in ? ldg_nc2(prm.scales + grow[b] + g) : uint16_t(0);
            bi[b][c] = in ? ldg_nc2(prm.biases + grow[b] + g) : uint16_t(0);
          }
      };
      // this warp's first K block of the tile: it0 + kb0 == h (mod H)
      const int kb0 = static_cast<int>((static_cast<uint32_t>(h) + H - it0 % H) % H);
      uint16_t sc_pf[2][2][CH], bi_pf[2][2][CH];
      load_sb(kb0, sc_pf[0], bi_pf[0]);
      load_sb(kb0 + H, sc_pf[1], bi_pf[1]);
      int slot = 0;
      for (int kb = kb0; kb < KB; kb += H, slot ^= 1) {
        const uint32_t it = it0 + kb;
        const int s = it % S;
        const uint32_t r = it / S;
        uint16_t sc[2][CH], bi[2][CH];
#pragma unroll
        for (int b = 0; b < WB; ++b)
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            sc[b][c] = sc_pf[slot][b][c];
            bi[b][c] = bi_pf[slot][b][c];
          }
        load_sb(kb + 2 * H, sc_pf[slot], bi_pf[slot]);
        if (!(ok = wait(&full[s], r & 1, abort_flag, kFaultDequantWait))) break;
        if (r >= 1 && !(ok = wait(&empty[s], (r - 1) & 1, abort_flag, kFaultDequantWait))) break;
        __syncwarp();  // lanes leave the spin at different times; tcgen05.st needs the whole warp
        const uint8_t *wtile = smem + s * C::STAGE_BYTES + C::X_BYTES;
        const uint32_t a_tmem = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::ACC_COLS + s * WB * C::A_COLS;
#pragma unroll
        for (int b = 0; b < WB; ++b) {
          const uint32_t *wrow = reinterpret_cast<const uint32_t *>(wtile) + (b * 128 + lrow) * C::BKW;
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
            uint32_t cols[16];
            dequant_chunk_f16<BITS>(w, sc[b][c], bi[b][c], cols);
            tmem_st16(a_tmem + b * C::A_COLS + c * 16, cols);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[s]);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      if (!(ok = wait(acc_full, t & 1, abort_flag, kFaultEpilogueWait))) break;
      if (!(ok = wait(&exp_ready[t & 1], (t >> 1) & 1, abort_flag, kFaultEpilogueWait))) break;
      __syncwarp();
      tc_fence_after();
      const float *upt = up + (t & 1) * kBN;
      // blocks of 32 accumulator columns (W blocks x 4 token blocks), dealt to the quadrant's warps
#pragma unroll 1
      for (int blk = h; blk < 4 * WB; blk += H) {
        const int b = blk >> 2, col = (blk & 3) * 32;
        uint32_t v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * kBN + col, v);
        tmem_ld_wait();
        if (rok[b]) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int m = m0 + col + i;
            if (m < prm.M)
              prm.y[static_cast<int64_t>(m) * prm.N + nr[b]] = __float2bfloat16_rn(__uint_as_float(v[i]) * upt[col + i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(acc_empty);
        mbar_arrive(&exp_free[t & 1]);
      }
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

template <int BITS, int WB>
cudaError_t launch_t(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                     const uint16_t *biases, int64_t N, int G, uint16_t *y, cudaStream_t stream) {
  using C = Cfg<BITS, WB>;
  constexpr int kWRows = C::WROWS;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap x_map, w_map;
  if (!encode_2d_cached(fn, &x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(K),
                        static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 64, kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int64_t P = K * BITS / 32;
  if (!encode_2d_cached(fn, &w_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, static_cast<uint64_t>(P),
                        static_cast<uint64_t>(N), static_cast<uint64_t>(P) * 4, C::BKW, kWRows,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  Params prm;
  prm.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  prm.scales = reinterpret_cast<const __half *>(scales);
  prm.biases = reinterpret_cast<const __half *>(biases);
  prm.y = reinterpret_cast<__nv_bfloat16 *>(y);
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.K = static_cast<int>(K);
  prm.G = G;
  prm.Gn = static_cast<int>(K / G);
  prm.m_tiles = static_cast<int>((M + kBN - 1) / kBN);
  prm.n_tiles = static_cast<int>((N + kWRows - 1) / kWRows);

  auto kern = qmm2_kernel<BITS, WB>;
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
  // the pre-kernel: one warp per token row
  const unsigned eblocks = static_cast<unsigned>((M + kExpThreads / 32 - 1) / (kExpThreads / 32));
  qmm2_exponents_kernel<<<eblocks, kExpThreads, 0, stream>>>(prm.x, prm.M, prm.K, prm.N, prm.n_tiles, kWRows,
                                                              reinterpret_cast<uint8_t *>(y));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>(prm.m_tiles) * prm.n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(tiles, sms)));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x_map, w_map, prm);
}

}  // namespace v2
}  // namespace qmm

// The workspace-free tensor-core matmul takes the shapes of the workspace one:
// K*bits a multiple of 128 (16-byte packed rows for TMA); K blocks past the end
// of a row are read as zeros by TMA (codes and activations alike).
bool qmm2_supports(int64_t M, int64_t N, int64_t K, int G, int bits) {
  (void)G;
  if (M <= 0 || N <= 0 || K <= 0) return false;
  return (K * bits) % 128 == 0;
}

// Tile height: two 128-row W blocks per CTA (each x tile feeds 256 rows) unless
// one block gives the grid a clearly better last wave (few tiles: small M and N).
static int pick_wblocks(int64_t M, int64_t N, int sms) {
  auto eff = [&](int64_t wrows) {
    const int64_t t = ((M + 127) / 128) * ((N + wrows - 1) / wrows);
    const int64_t waves = (t + sms - 1) / sms;
    return static_cast<double>(t) / static_cast<double>(waves * sms);
  };
  return eff(128) > eff(256) + 0.05 ? 1 : 2;
}

template <int BITS>
static cudaError_t launch_bits2(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                                const uint16_t *biases, int64_t N, int G, uint16_t *y, cudaStream_t s) {
  static thread_local int cached_dev = -1, sms = 148;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cached_dev = dev;
  }
  if (pick_wblocks(M, N, sms) == 1) return qmm::v2::launch_t<BITS, 1>(x, M, K, packed, scales, biases, N, G, y, s);
  return qmm::v2::launch_t<BITS, 2>(x, M, K, packed, scales, biases, N, G, y, s);
}

cudaError_t launch_qmm2(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
                        const uint16_t *biases, int64_t N, int G, int bits, uint16_t *y, cudaStream_t s) {
  switch (bits) {
    case 2: return launch_bits2<2>(x, M, K, packed, scales, biases, N, G, y, s);
    case 3: return launch_bits2<3>(x, M, K, packed, scales, biases, N, G, y, s);
    case 4: return launch_bits2<4>(x, M, K, packed, scales, biases, N, G, y, s);
    default: return launch_bits2<8>(x, M, K, packed, scales, biases, N, G, y, s);
  }
}

cudaError_t read_and_clear_qmm2_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_qmm2_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_qmm2_fault, &zero, sizeof(uint32_t));
}

}  // namespace aq
