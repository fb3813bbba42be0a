// QMV on the 5th-generation tensor cores (tcgen05 + tensor memory), sm_100a:
// y[M,N] = x[M,K] . dequant(W)^T for decode, M = 1..8 activation rows, affine
// 2/4/8-bit codes, W never materialised.
//
// Method: metalworking "MLX Quantization", section "Mechanics" (QMV streams
// each weight once per decode step; multi-token decode, M = 3..6, must still
// read W once) and anllm "Tutorial 10: Quantization", section 5 (y = x @ W^T on
// the packed weights).  Per group g of a row: y += s_g * sum_k q_k x_k +
// b_g * sum_k x_k.
//
// Arithmetic (as the mma.sync decode kernel in qmv_tc.cu): each group's
// activations enter as 16-bit fixed point, x_int = rint(x * 2^e) with 2^e the
// power of two that puts the group's largest |x| in [2^13, 2^14); x_int is
// split into two signed bytes, x_int = 256 * hi + lo with lo in [-128, 127]
// and hi in [-64, 64].  The codes enter as unsigned bytes.  Per group the
// integer sums sum q*lo and sum q*hi are exact (int32); the fold applies
// scale * 2^-e and the bias term in fp32.
//
// B200 design:
//  * A CTA owns 128 rows of W (TMEM lane = row) and a range of K; when there
//    are few row tiles, a cluster of C CTAs splits K and the partial sums meet
//    in distributed shared memory (no workspace).
//  * Warp 0 (one lane): TMA producer, 128 rows x Kc codes per stage into a
//    ring of shared-memory stages.  Each box is 16 bytes wider than a stage's
//    codes, so a warp's 16-byte reads of 8 consecutive rows hit all 32 banks.
//  * Warps 2..17 (four per TMEM lane quadrant, taking stages in turn, each with
//    its own TMEM stage): first
//    stage this CTA's activations as the MMA's B operand (16 rows: token m's
//    low digits in row 2m, high digits in row 2m + 1; 128-byte swizzled
//    K-major), then per stage unpack their row's codes into bytes (three
//    logic ops per 8 codes at 4 bits) and write them with tcgen05.st into a
//    TMEM stage, the MMA's A operand; once the stage's MMAs are done, read its
//    per-group accumulators back with tcgen05.ld and fold them.  The four
//    workers of a quadrant overlap one another's MMA round trips.
//  * Warp 1 (one lane): tcgen05.mma.kind::i8 (u8 codes x s8 digits, int32
//    accumulate, M = 128, N = 16, K = 32), one accumulator per group, so 1 to 8
//    tokens cost the same MMAs; warp 1 also owns the TMEM allocation.
//  * Every wait on a barrier is bounded; a timeout sets a bit of the fault
//    word, the CTA stops issuing work, waits for its copies and MMAs in flight
//    and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "tc05.cuh"

namespace aq {

__device__ uint32_t g_qmv5_fault = 0;

namespace qmm {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();  // driver entry point, resolved once (qmm.cu)
}

namespace u5 {

constexpr int kRows = 128;
constexpr int kWorkerWarp0 = 2;
constexpr int kWorkersPerQuad = 4;  // each owns one TMEM stage: four stages in flight per quadrant
constexpr int kWorkers = 4 * kWorkersPerQuad;
constexpr int kThreads = 32 * (kWorkerWarp0 + kWorkers);
constexpr int kTmemCols = 512;
constexpr int kNT = kWorkersPerQuad;  // TMEM stages, one per worker of a quadrant
constexpr int kBRows = 16;   // B rows: 8 tokens x 2 digits
constexpr int kSmemBudget = 224 * 1024;

struct Args {
  const __nv_bfloat16 *x;
  const __half *scales, *biases;
  __nv_bfloat16 *y;
  int M, N, K, Gn;
  int C;          // CTAs per row tile (cluster size); each takes Kr of K
  int Kr;         // K of one CTA (a multiple of Kc)
  int Kc;         // codes of a row per stage
  int nst;        // stages per CTA
  int NS;         // shared-memory ring depth (a multiple of kWorkersPerQuad)
  int pitch;      // bytes per row in a stage (the TMA box width)
  int stage_bytes;
  int b_off, tab_off, red_off, bar_off;
  int early_w;    // stages issued before the previous kernel has completed (overlap mode)
  long long wait_cycles;
  int stall;      // nonzero: the workers also wait on a barrier nothing completes (timeout test)
};

AQ_DEVICE bool wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, long long limit) {
  return aq::mbar_wait(bar, parity, abort_flag, &g_qmv5_fault, kFaultQmvWait, limit);
}

// D[tmem] (+)= A[tmem] (u8) * B[smem desc]^T (s8), int32 accumulate.
AQ_DEVICE void mma_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::i8: D = s32 (2), A = u8 (0), B = s8 (1), both
// K-major, M = 128, N = 16.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

AQ_DEVICE void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// The first 2*MP accumulator columns of a group (tokens 0..MP-1, two digits each).
template <int MP>
AQ_DEVICE void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[2 * MP]) {
  if constexpr (MP == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr)
                 : "memory");
  } else if constexpr (MP == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr)
                 : "memory");
  } else if constexpr (MP == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
  }
}

// Slot (K position inside the MMA operands) of code c of a word-aligned run:
// unpacking takes every (8/bits)-th code into one byte lane, so 4-bit codes
// 0..7 of a word sit at slots 0,4,1,5,2,6,3,7 -> slot(c) = (c % 2) * 4 + c / 2,
// 2-bit codes 0..15 at slot (c % 4) * 4 + c / 4, 8-bit codes in order.
template <int BITS>
__host__ __device__ constexpr int code_slot(int c) {
  return BITS == 4 ? (c % 2) * 4 + c / 2 : BITS == 2 ? (c % 4) * 4 + c / 4 : c;
}

// Byte offset inside B of (row n, K position k) in the 128-byte swizzled
// K-major layout: atoms of 8 rows x 128 bytes, two atoms (16 rows) per 128 K.
AQ_DEVICE int b_offset(int n, int k) {
  const int b = k & 127;
  return (k >> 7) * (kBRows * 128) + (n >> 3) * 1024 + (n & 7) * 128 + ((((b >> 4) ^ (n & 7))) << 4) + (b & 15);
}

AQ_DEVICE void mapa_and_load(uint32_t local, uint32_t rank, float &v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
}

AQ_DEVICE void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int BITS, int G, int MP>
__global__ void __launch_bounds__(kThreads, 1) qmv_umma_kernel(const __grid_constant__ Args a,
                                                               const __grid_constant__ CUtensorMap wmap) {
  constexpr int SZ = BITS == 2 ? 16 : 8;  // activation elements one staging lane takes (one run of slots)
  constexpr int L = G / SZ;               // staging lanes per (token, group)
  static_assert(L >= 2 && L <= 16 && (L & (L - 1)) == 0, "staging lanes per group");
  static_assert(BITS == 8 || SZ == 32 / BITS, "a staging run is one word of codes");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  uint8_t *bmat = smem + a.b_off;
  float4 *tab = reinterpret_cast<float4 *>(smem + a.tab_off);  // [MP][Gr]: (sum x, 2^-e_lo, 2^-e_hi, 0)
  float *red = reinterpret_cast<float *>(smem + a.red_off);    // [kWorkersPerQuad][kRows][MP]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + a.bar_off);
  uint64_t *empty = full + a.NS;
  uint64_t *a_full = empty + a.NS;
  uint64_t *mma_done = a_full + kNT;
  uint64_t *b_ready = mma_done + kNT;
  uint64_t *stall_bar = b_ready + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(stall_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *issued_ctr = reinterpret_cast<int *>(tmem_slot + 2);
  int *mma_ctr = issued_ctr + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x / a.C;
  const int rank = blockIdx.x - tile * a.C;  // == the CTA's rank in its cluster (cluster dims (C, 1, 1))
  const int row0 = tile * kRows;
  const int k0 = rank * a.Kr;                // first K position of this CTA
  const int Gr = a.Kr / G;                   // groups of a row in this CTA
  const int GPS = a.Kc / G;                  // groups per stage
  const int ACOLS = a.Kc / 4;                // TMEM columns of one A stage
  const long long wlim = a.wait_cycles;

  if (tid == 0) {
    for (int s = 0; s < a.NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);  // the four worker warps (one per quadrant) that take the stage
    }
    for (int t = 0; t < kNT; ++t) {
      mbar_init(&a_full[t], 4);
      mbar_init(&mma_done[t], 1);
    }
    mbar_init(b_ready, kWorkers);
    mbar_init(stall_bar, 1);
    *abort_flag = 0;
    *issued_ctr = 0;
    *mma_ctr = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  qmm::tc_fence_before();
  __syncthreads();
  qmm::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (a.C > 1) cluster_sync();  // the cluster's barriers and shared memory exist before any remote access
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // TMEM: A stage t at columns t * ACOLS; its accumulators (GPS groups x 16
  // columns) from column kNT * ACOLS + t * GPS * 16.
  auto a_col = [&](int t) { return static_cast<uint32_t>(t * ACOLS); };
  auto acc_col = [&](int t) { return static_cast<uint32_t>(kNT * ACOLS + t * GPS * 16); };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
      const int wstep = a.Kc * BITS / 32;  // words of a row per stage
      const int kw0 = k0 * BITS / 32;
      auto issue = [&](int st) {
        const int s = st % a.NS;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kRows * a.pitch));
        tma_load_2d(ring + static_cast<size_t>(s) * a.stage_bytes, &wmap, &full[s], kw0 + st * wstep, row0);
      };
      // the weights are not written by the kernel this launch may overlap, so
      // up to the whole ring goes out before waiting for it
      const int early = std::min(std::min(a.nst, a.NS), a.early_w);
      int st = 0;
      for (; st < early; ++st) issue(st);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (; st < std::min(a.nst, a.NS); ++st) issue(st);
      for (; st < a.nst; ++st) {
        const int s = st % a.NS;
        if (!wait(&empty[s], ((st / a.NS) - 1) & 1, abort_flag, wlim)) break;
        issue(st);
      }
      *issued_ctr = st;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t b_base = smem_u32(bmat);
      int st = 0;
      if (wait(b_ready, 0, abort_flag, wlim)) {
        for (; st < a.nst; ++st) {
          const int t = st % kNT;
          if (!wait(&a_full[t], (st / kNT) & 1, abort_flag, wlim)) break;
          qmm::tc_fence_after();
          for (int j = 0; j < GPS; ++j) {
#pragma unroll
            for (int ks = 0; ks < G / 32; ++ks) {
              const int kk = st * a.Kc + j * G + ks * 32;  // K position inside this CTA's range
              const uint32_t baddr = b_base + (kk >> 7) * (kBRows * 128) + (kk & 127);
              mma_i8(tmem_base + acc_col(t) + j * 16, tmem_base + a_col(t) + (j * (G / 32) + ks) * 8,
                     qmm::sw128_kmajor_desc(baddr), kIdesc, ks > 0 ? 1u : 0u);
            }
          }
          qmm::tc_commit(&mma_done[t]);
        }
      }
      *mma_ctr = st;
    }
  } else {
    // ------------------------------------------------------------------ workers
    const int wk = warp - kWorkerWarp0;       // 0..15
    const int q = warp & 3;                   // TMEM lane quadrant this warp may access
    const int h = wk >> 2;                    // takes the stages st with st % kWorkersPerQuad == h (TMEM stage h)
    const int wt = wk * 32 + lane;            // index among the workers
    constexpr int WT = kWorkers * 32;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // x may be the previous kernel's output

    // ---- B: zero it all (rows of absent tokens must be zero), then the digits
    {
      const int nb16 = kBRows * a.Kr / 16;
      for (int i = wt; i < nb16; i += WT) reinterpret_cast<uint4 *>(bmat)[i] = make_uint4(0u, 0u, 0u, 0u);
      asm volatile("bar.sync 1, %0;" ::"n"(WT) : "memory");
      const int items = a.M * Gr * L;  // (token, group, lane of the group's run)
      for (int i0 = 0; i0 < items; i0 += WT) {
        const int i = i0 + wt;
        const bool act = i < items;
        const int ii = act ? i : 0;
        const int part = ii % L, mg = ii / L;
        const int m = mg / Gr, g = mg - m * Gr;
        const int kl = g * G + part * SZ;  // K position (in this CTA's range) of the run
        float v[SZ];
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(m) * a.K + k0 + kl);
#pragma unroll
        for (int c = 0; c < SZ / 8; ++c) {
          const uint4 u = act ? ldg_nc16(src + c) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[8 * c + 2 * j] = bf16_bits_to_float(w4[j] & 0xFFFFu);
            v[8 * c + 2 * j + 1] = bf16_bits_to_float(w4[j] >> 16);
          }
        }
        float amax = 0.0f, sx = 0.0f;
#pragma unroll
        for (int j = 0; j < SZ; ++j) {
          amax = fmaxf(amax, fabsf(v[j]));
          sx += v[j];
        }
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {  // the group's L lanes are consecutive (L divides 32)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          sx += __shfl_xor_sync(0xffffffffu, sx, o);
        }
        // 2^e with the group's largest |x| * 2^e in [2^13, 2^14) (e within normal fp32 powers)
        int e = 0;
        if (amax > 0.0f) {
          const int be = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
          e = min(max(13 - (be == 0 ? -127 : be - 127), -126), 126);
        }
        const int e_hi = e >> 1, e_lo = e - e_hi;
        const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
        // digits: x_int = rint(v * 2^e) in [-2^14, 2^14]; lo = x_int's low byte as a
        // signed value, hi = (x_int - lo) / 256 in [-64, 64]
        uint8_t lo[SZ], hi[SZ];
#pragma unroll
        for (int j = 0; j < SZ; ++j) {
          const int xi = __float2int_rn(v[j] * sc);
          const int l8 = static_cast<int>(static_cast<int8_t>(xi & 0xFF));
          lo[j] = static_cast<uint8_t>(l8);
          hi[j] = static_cast<uint8_t>((xi - l8) >> 8);
        }
        if (act) {
          // the run is one word's codes (2 and 4 bits) or two words (8 bits):
          // element j goes to slot code_slot(j) of the run
          uint8_t plo[SZ], phi[SZ];
#pragma unroll
          for (int j = 0; j < SZ; ++j) {
            plo[code_slot<BITS>(j)] = lo[j];
            phi[code_slot<BITS>(j)] = hi[j];
          }
#pragma unroll
          for (int h16 = 0; h16 < SZ / 8; ++h16) {
            uint32_t wl[2], wh[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              wl[z] = plo[8 * h16 + 4 * z] | (plo[8 * h16 + 4 * z + 1] << 8) | (plo[8 * h16 + 4 * z + 2] << 16) |
                      (static_cast<uint32_t>(plo[8 * h16 + 4 * z + 3]) << 24);
              wh[z] = phi[8 * h16 + 4 * z] | (phi[8 * h16 + 4 * z + 1] << 8) | (phi[8 * h16 + 4 * z + 2] << 16) |
                      (static_cast<uint32_t>(phi[8 * h16 + 4 * z + 3]) << 24);
            }
            *reinterpret_cast<uint2 *>(bmat + b_offset(2 * m, kl + 8 * h16)) = make_uint2(wl[0], wl[1]);
            *reinterpret_cast<uint2 *>(bmat + b_offset(2 * m + 1, kl + 8 * h16)) = make_uint2(wh[0], wh[1]);
          }
          if (part == 0)
            tab[m * Gr + g] = make_float4(sx, __uint_as_float(static_cast<uint32_t>(127 - e_lo) << 23),
                                          __uint_as_float(static_cast<uint32_t>(127 - e_hi) << 23), 0.0f);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B is read by the tensor core
      asm volatile("bar.sync 1, %0;" ::"n"(WT) : "memory");  // every worker reads the whole table in its folds
      if (lane == 0) mbar_arrive(b_ready);
    }
    // timeout test: a wait on a barrier nothing completes runs out and raises the abort flag
    if (a.stall) wait(stall_bar, 0, abort_flag, wlim);

    const int r = q * 32 + lane;  // this thread's row of the tile (TMEM lane)
    const int n = row0 + r;
    const bool row_ok = n < a.N;
    const int64_t gbase = static_cast<int64_t>(row_ok ? n : 0) * a.Gn + k0 / G;
    float yacc[MP];
#pragma unroll
    for (int m = 0; m < MP; ++m) yacc[m] = 0.0f;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);

    // fold: the stage's per-group accumulators, read in batches of GB groups
    // (one wait per batch), into this row's partial sums
    constexpr int GB = 2 * MP * 4 <= 32 ? 4 : 2;
    auto fold = [&](int st, const __half (&sc)[8], const __half (&bi)[8]) -> bool {
      const int t = st % kNT;
      if (!wait(&mma_done[t], (st / kNT) & 1, abort_flag, wlim)) return false;
      qmm::tc_fence_after();
      for (int j0 = 0; j0 < GPS; j0 += GB) {
        uint32_t v[GB][2 * MP];
#pragma unroll
        for (int jj = 0; jj < GB; ++jj)
          if (j0 + jj < GPS) tmem_ld_cols<MP>(lane_base + acc_col(t) + (j0 + jj) * 16, v[jj]);
        qmm::tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < GB; ++jj) {
          const int j = j0 + jj;
          if (j >= GPS) break;
          const float s = __half2float(sc[j]), b = __half2float(bi[j]);
          const int g = st * GPS + j;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            if (m < a.M) {
              const float4 T = tab[m * Gr + g];
              const float D =
                  static_cast<float>(static_cast<int>(v[jj][2 * m]) + 256 * static_cast<int>(v[jj][2 * m + 1]));
              yacc[m] = fmaf(s * T.z, D * T.y, fmaf(b, T.x, yacc[m]));
            }
          }
        }
      }
      return true;
    };

    bool ok = true;
    __half sc_cur[8], bi_cur[8];
    for (int st = h; st < a.nst; st += kWorkersPerQuad) {
      const int s = st % a.NS, t = st % kNT;  // t == h: this worker's TMEM stage
      // this stage's scales and biases (used by the fold below)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool in = j < GPS && row_ok;
        sc_cur[j] = in ? __ldg(a.scales + gbase + st * GPS + j) : __float2half(0.0f);
        bi_cur[j] = in ? __ldg(a.biases + gbase + st * GPS + j) : __float2half(0.0f);
      }
      if (!(ok = wait(&full[s], (st / a.NS) & 1, abort_flag, wlim))) break;
      __syncwarp();
      // unpack this row's codes into bytes, 32 codes (8 TMEM columns) at a time
      // (the TMEM stage is free: this warp folded its previous stage, whose MMAs were done)
      const uint32_t *wr = reinterpret_cast<const uint32_t *>(ring + static_cast<size_t>(s) * a.stage_bytes +
                                                               static_cast<size_t>(r) * a.pitch);
      for (int ks = 0; ks < a.Kc / 32; ++ks) {
        uint32_t cols[8];
        if constexpr (BITS == 4) {
          const uint4 u = reinterpret_cast<const uint4 *>(wr)[ks];
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            cols[2 * i] = w4[i] & 0x0F0F0F0Fu;
            cols[2 * i + 1] = (w4[i] >> 4) & 0x0F0F0F0Fu;
          }
        } else if constexpr (BITS == 8) {
          const uint4 u0 = reinterpret_cast<const uint4 *>(wr)[2 * ks];
          const uint4 u1 = reinterpret_cast<const uint4 *>(wr)[2 * ks + 1];
          cols[0] = u0.x; cols[1] = u0.y; cols[2] = u0.z; cols[3] = u0.w;
          cols[4] = u1.x; cols[5] = u1.y; cols[6] = u1.z; cols[7] = u1.w;
        } else {
          const uint2 u = reinterpret_cast<const uint2 *>(wr)[ks];
          const uint32_t w2[2] = {u.x, u.y};
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            cols[4 * i] = w2[i] & 0x03030303u;
            cols[4 * i + 1] = (w2[i] >> 2) & 0x03030303u;
            cols[4 * i + 2] = (w2[i] >> 4) & 0x03030303u;
            cols[4 * i + 3] = (w2[i] >> 6) & 0x03030303u;
          }
        }
        tmem_st8(lane_base + a_col(t) + ks * 8, cols);
      }
      qmm::tmem_st_wait();
      qmm::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[t]);
        mbar_arrive(&empty[s]);
      }
      if (!(ok = fold(st, sc_cur, bi_cur))) break;
    }
    // the warps of a quadrant: sum their partials (in worker order)
#pragma unroll
    for (int m = 0; m < MP; ++m) red[(h * kRows + r) * MP + m] = yacc[m];
    asm volatile("bar.sync 1, %0;" ::"n"(WT) : "memory");
    if (h == 0) {
#pragma unroll
      for (int m = 0; m < MP; ++m) {
        float sum = yacc[m];
        for (int w = 1; w < kWorkersPerQuad; ++w) sum += red[(w * kRows + r) * MP + m];
        red[r * MP + m] = sum;
      }
    }
  }

  // ---- end: every thread of every CTA of the cluster comes here
  __syncthreads();
  if (a.C > 1) {
    cluster_sync();  // every rank's partial sums are in its own red[0]
    if (rank == 0 && warp >= kWorkerWarp0 && (warp - kWorkerWarp0) < 4) {
      const int r = (warp & 3) * 32 + lane;
      const int n = row0 + r;
      for (int m = 0; m < a.M; ++m) {
        float sum = red[r * MP + m];
        for (int c = 1; c < a.C; ++c) {
          float pv;
          mapa_and_load(smem_u32(red + r * MP + m), static_cast<uint32_t>(c), pv);
          sum += pv;
        }
        if (n < a.N) a.y[static_cast<int64_t>(m) * a.N + n] = __float2bfloat16_rn(sum);
      }
    }
    cluster_sync();  // no CTA leaves while rank 0 may still read its shared memory
  } else if (warp >= kWorkerWarp0 && (warp - kWorkerWarp0) < 4) {
    const int r = (warp & 3) * 32 + lane;
    const int n = row0 + r;
    if (n < a.N)
      for (int m = 0; m < a.M; ++m) a.y[static_cast<int64_t>(m) * a.N + n] = __float2bfloat16_rn(red[r * MP + m]);
  }
  // after an abort: copies and MMAs still in flight land before the CTA exits
  if (tid == 0 && *abort_flag) {
    const int issued = *issued_ctr;
    for (int j = std::max(0, issued - a.NS); j < issued; ++j) mbar_drain(&full[j % a.NS], (j / a.NS) & 1);
    const int mm = *mma_ctr;
    if (mm > 0) mbar_drain(&mma_done[(mm - 1) % kNT], ((mm - 1) / kNT) & 1);
  }
  qmm::tc_fence_before();
  __syncthreads();
  qmm::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host plan
// ---------------------------------------------------------------------------
struct Plan {
  Args a;
  int grid;
  size_t smem;
};

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

static bool make_plan(int64_t M, int64_t N, int64_t K, int G, int bits, int sms, Plan &pl) {
  if (!(bits == 2 || bits == 4 || bits == 8) || !(G == 32 || G == 64 || G == 128)) return false;
  if (M < 1 || M > 8 || N < 1 || K < 1 || N >= (int64_t(1) << 30) || K >= (int64_t(1) << 30)) return false;
  const int Kc = G == 32 ? 128 : 256;
  if (K % Kc != 0) return false;
  const int MP = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  const int64_t T = (N + kRows - 1) / kRows;
  // K split across a cluster when there are few row tiles
  int C = 1;
  while (C < 8 && T * C * 2 <= sms + sms / 4 && (K / Kc) % (2 * C) == 0) C *= 2;
  Args &a = pl.a;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.Gn = static_cast<int>(K / G);
  a.C = C;
  a.Kc = Kc;
  a.Kr = static_cast<int>(K / C);
  a.nst = a.Kr / Kc;
  a.pitch = Kc * bits / 8 + 16;  // bytes per row in a stage: 16 more than the codes (bank spread)
  a.stage_bytes = static_cast<int>(round_up(static_cast<int64_t>(kRows) * a.pitch, 1024));
  a.early_w = 0;
  a.wait_cycles = kWaitCycles;
  a.stall = 0;
  a.x = nullptr;
  a.scales = a.biases = nullptr;
  a.y = nullptr;
  const int64_t Gr = a.Kr / G;
  const int64_t b_bytes = static_cast<int64_t>(kBRows) * a.Kr;
  const int64_t tab_bytes = static_cast<int64_t>(MP) * Gr * 16;
  const int64_t red_bytes = static_cast<int64_t>(kWorkersPerQuad) * kRows * MP * 4;
  auto total = [&](int ns) {
    int64_t off = static_cast<int64_t>(ns) * a.stage_bytes;
    off = round_up(off, 1024) + b_bytes;
    off = round_up(off, 16) + tab_bytes + red_bytes;
    off = round_up(off, 8) + (2 * ns + 2 * kNT + 2) * 8 + 16;
    return off + 1024;  // alignment slack of the dynamic shared memory base
  };
  int ns = 0;
  for (int c = kWorkersPerQuad; c <= 16; c += kWorkersPerQuad)
    if (total(c) <= kSmemBudget) ns = c;
  if (ns == 0) return false;
  a.NS = ns;
  int64_t off = static_cast<int64_t>(ns) * a.stage_bytes;
  a.b_off = static_cast<int>(round_up(off, 1024));
  off = a.b_off + b_bytes;
  a.tab_off = static_cast<int>(round_up(off, 16));
  a.red_off = static_cast<int>(a.tab_off + tab_bytes);
  a.bar_off = static_cast<int>(round_up(a.red_off + red_bytes, 8));
  pl.smem = static_cast<size_t>(total(ns));
  pl.grid = static_cast<int>(T * C);
  // TMEM: kNT stages of A (Kc/4 columns) and accumulators (16 per group)
  if (kNT * (Kc / 4 + (Kc / G) * 16) > kTmemCols) return false;
  if (a.pitch / 4 > 256) return false;  // TMA box width (32-bit elements)
  return true;
}

static std::atomic<long long> g_limit{kWaitCycles};
static std::atomic<bool> g_stall{false};

template <int BITS, int G, int MP>
static cudaError_t launch(const Plan &pl, const CUtensorMap &wmap, bool overlap, cudaStream_t stream) {
  auto kern = qmv_umma_kernel<BITS, G, MP>;
  static thread_local int cached_dev = -1;
  static thread_local size_t cached_smem = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev || pl.smem > cached_smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem))) !=
        cudaSuccess)
      return e;
    if (pl.a.C > 1 &&
        (e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
      return e;
    cached_dev = dev;
    cached_smem = pl.smem;
  }
  Args a = pl.a;
  a.early_w = overlap ? a.NS : 0;
  a.wait_cycles = g_limit.load(std::memory_order_relaxed);
  a.stall = g_stall.load(std::memory_order_relaxed) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pl.a.C > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = pl.a.C;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (overlap) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, a, wmap);
}

template <int BITS, int G>
static cudaError_t launch_mp(const Plan &pl, const CUtensorMap &wmap, bool overlap, cudaStream_t s) {
  switch (pl.a.M <= 1 ? 1 : pl.a.M <= 2 ? 2 : pl.a.M <= 4 ? 4 : 8) {
    case 1: return launch<BITS, G, 1>(pl, wmap, overlap, s);
    case 2: return launch<BITS, G, 2>(pl, wmap, overlap, s);
    case 4: return launch<BITS, G, 4>(pl, wmap, overlap, s);
    default: return launch<BITS, G, 8>(pl, wmap, overlap, s);
  }
}

template <int BITS>
static cudaError_t launch_g(const Plan &pl, const CUtensorMap &wmap, int G, bool overlap, cudaStream_t s) {
  switch (G) {
    case 32: return launch_mp<BITS, 32>(pl, wmap, overlap, s);
    case 64: return launch_mp<BITS, 64>(pl, wmap, overlap, s);
    default: return launch_mp<BITS, 128>(pl, wmap, overlap, s);
  }
}

}  // namespace u5

bool qmv_umma_supported(int64_t M, int64_t N, int64_t K, int G, int bits) {
  u5::Plan pl;
  return u5::make_plan(M, N, K, G, bits, 148, pl);
}

cudaError_t launch_qmv_umma(const uint16_t *x, int64_t M, int64_t K, const uint32_t *packed, const uint16_t *scales,
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
  u5::Plan pl;
  if (!u5::make_plan(M, N, K, G, bits, sms, pl)) return cudaErrorInvalidValue;
  pl.a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
  pl.a.scales = reinterpret_cast<const __half *>(scales);
  pl.a.biases = reinterpret_cast<const __half *>(biases);
  pl.a.y = reinterpret_cast<__nv_bfloat16 *>(y);
  auto fn = qmm::encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap wmap;
  const int64_t words = K * bits / 32;
  if (!encode_2d_cached(fn, &wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, static_cast<uint64_t>(words),
                        static_cast<uint64_t>(N), static_cast<uint64_t>(words) * 4,
                        static_cast<uint32_t>(pl.a.pitch / 4), static_cast<uint32_t>(u5::kRows),
                        CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const bool overlap = (flags & AQ_MATMUL_OVERLAP_PREVIOUS) != 0;
  switch (bits) {
    case 2: return u5::launch_g<2>(pl, wmap, G, overlap, s);
    case 4: return u5::launch_g<4>(pl, wmap, G, overlap, s);
    default: return u5::launch_g<8>(pl, wmap, G, overlap, s);
  }
}

void set_qmv_umma_wait_limit(long long cycles) { u5::g_limit.store(cycles > 0 ? cycles : kWaitCycles); }
void set_qmv_umma_wait_stall(bool on) { u5::g_stall.store(on); }

cudaError_t read_and_clear_qmv5_fault(uint32_t *word) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_qmv5_fault, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  return cudaMemcpyToSymbol(g_qmv5_fault, &zero, sizeof(uint32_t));
}

}  // namespace aq
