// mxfp8_gemm.cu -- a block-scaled MXFP8 x MXFP8 GEMM on the 5th-generation
// tensor cores (tcgen05, kind::mxf8f6f4.block_scale), the consumer of the
// quantizer's codes and 128x4-tile swizzled E8M0 scales, for sm_100a.
//
//   D[m, n] = sum_k decode(A[m, k]) 2^(SA[m, k/32] - 127)
//                 * decode(B[n, k]) 2^(SB[n, k/32] - 127)
//
// A [M, K] and B [N, K] are E4M3 codes as mxfp8_quantize writes them (rows of
// K contiguous bytes: both operands K-major, B in the [out, in] layout of a
// linear layer's weight), SA / SB their scales in the swizzled layout
// (mxfp8_quantize's scale_swz). The products of two E4M3 values and two
// power-of-two scales are exact; the tensor core accumulates them in fp32.
// Context: "V4 mxfp4 #1372" (description: block-scaled low-precision GEMMs
// reading E8M0 scales on Blackwell) and "PR #1935 完整报告 -- Use
// TransformerEngine for MXFP8 quantization" (the quantized weights feed the
// GEMM); the scale-tile layout is the one the block-scaled MMA reads.
//
// Two kernels. When M and N both exceed 128, CTA pairs (clusters of two, one
// CTA per SM) walk 256 x 256 output tiles with the pair form of the MMA; it is
// described with mxfp8_gemm_pair_kernel below. Otherwise the single-CTA
// kernel runs.
//
// Single-CTA structure: persistent CTAs (one per multiprocessor) walk
// 128 x BN output tiles (BN = 256, or 128 when N <= 128) with six warps:
//  - warp 0, one lane: producer. Per K block of 128: TMA loads of the A tile
//    (128 rows x 128 bytes) and the B tile (BN rows x 128 bytes), both with
//    the 128-byte swizzle, and bulk copies of the 512-byte scale tiles (one
//    for A, BN / 128 for B) into the next shared-memory stage; completion is
//    counted in bytes on the stage's "full" mbarrier. The stages run on
//    across tiles, so the next tile's loads overlap this tile's epilogue.
//  - warp 1, one lane: MMA issuer. Waits until the epilogue has read the
//    previous tile's accumulator ("acc_empty"), then per stage copies the
//    scale tiles into tensor memory (tcgen05.cp 32x128b.warpx4, the 32 x
//    16-byte scale tile broadcast to the four lane quarters), issues four
//    MMAs of K = 32 (one scale column each, selected by the scale-factor id;
//    M = 128, N = BN) and commits the stage's "empty" mbarrier; after the
//    tile's last stage it commits "acc_full".
//  - warps 2-5: epilogue. Each reads its quarter of the accumulator lanes
//    (tcgen05.ld 32x32b, warp w takes lanes 32 (w % 4) ..), hands the
//    accumulator back once the last columns are in registers, and writes its
//    rows of D as bf16 or fp32 while the next tile's MMAs run.
// Tensor memory: BN columns of fp32 accumulator plus 4 scale columns per
// 128-row scale tile and stage (4 for A, 4 or 8 for B).
//
// Every wait on an mbarrier gives up after about one second (by %globaltimer,
// from the start of that wait) or 2^30 polls; the kernel then records an
// error code in *err (when err is not NULL), skips the remaining work, frees
// its tensor memory and returns.
#include "common.cuh"
#include "tma.cuh"

namespace mxq {
namespace {

constexpr int kBM = 128, kBK = 128;  // kBK elements = bytes of E4M3
constexpr int kEpilogueWarps = 4;
constexpr int kGemmThreads = 32 * (2 + kEpilogueWarps);  // producer, MMA, epilogue warps
constexpr uint32_t kSfTile = 512;    // one 128 x 4 scale tile
constexpr uint32_t kBarBytes = 256;
// bf16 epilogue staging per warp: 32 rows x 64 columns (128 bytes), pitch 144
constexpr uint32_t kEpiPitch = 144;
constexpr uint32_t kEpiStageBytes = 32 * kEpiPitch;
constexpr uint64_t kWaitNs = 1000000000ull;  // one second

template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 128 ? 6 : 4;
  static constexpr uint32_t kTileA = kBM * kBK;                   // 16 KiB
  static constexpr uint32_t kTileB = BN * kBK;                    // 16 or 32 KiB
  static constexpr uint32_t kSfbTiles = BN / 128;
  static constexpr uint32_t kStageBytes =                         // a multiple of 1 KiB
      (kTileA + kTileB + kSfTile * (1 + kSfbTiles) + 1023u) & ~1023u;
  static constexpr uint32_t kSfColsPerStage = 4 * (1 + kSfbTiles);
  static constexpr uint32_t kTmemCols = BN + kStages * kSfColsPerStage <= 256 ? 256 : 512;
  static constexpr uint32_t kSmemBytes =
      kStages * kStageBytes + kBarBytes + kEpiStageBytes * kEpilogueWarps + 1024;  // + alignment slack
  static_assert(BN + kStages * kSfColsPerStage <= 512, "tensor memory");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

enum GemmError : int32_t { kErrNone = 0, kErrFullWait = 1, kErrEmptyWait = 2, kErrAccumWait = 3 };

struct GemmArgs {
  const uint8_t* sfa;   // swizzled scales of A
  const uint8_t* sfb;   // swizzled scales of B
  void* d;              // [M, N] row-major
  int32_t* err;         // device error word or NULL
  uint32_t M, N;
  uint32_t nk;          // K blocks of 128
  uint32_t kp4;         // 4-column scale tiles per 128-row block: ceil(K / 128)
  uint32_t nb128;       // 128-row blocks of B's scales: ceil(N / 128)
  uint32_t n_tiles_n;   // output tiles along N
  uint32_t ntiles;      // output tiles
};

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets in 16-byte units, descriptor version 1, layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return uint64_t((addr >> 4) & 0x3fffu) | (uint64_t(lbo & 0x3fffu) << 16) |
         (uint64_t(sbo & 0x3fffu) << 32) | (1ull << 46) | (uint64_t(layout) << 61);
}

// K-major operand tile, rows of 128 bytes with the 128-byte swizzle: 8-row
// groups 1024 bytes apart (layout type 2).
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) {
  return smem_desc(addr, 1, 1024 >> 4, 2);
}

// The 512-byte scale tile seen as 32 rows of 16 bytes, no swizzle.
__device__ __forceinline__ uint64_t scale_desc(uint32_t addr) {
  return smem_desc(addr, 1, 128 >> 4, 0);
}

// Instruction descriptor of kind::mxf8f6f4.block_scale: E4M3 x E4M3, both
// K-major, fp32 accumulator, M = 128, N = BN, E8M0 scales; the scale-factor
// ids pick byte `k` (the scale column of the k-th MMA of a K block) of the
// 32-bit scale columns of A and B.
template <int BN>
__device__ __forceinline__ uint32_t instr_desc(uint32_t k) {
  return (k << 4) | (uint32_t(BN >> 3) << 17) | (1u << 23) | (uint32_t(kBM >> 4) << 24) | (k << 29);
}

// The MMA, the scale copy and the commit for a converged warp: each is
// issued by the one lane that elect.sync picks, inside the same asm block.
// The MMA and the copy take their shared-memory descriptors as 32-bit words
// (low words of A and B, one high word), so the warp only adds offsets to
// precomputed words.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p, e; .reg .b64 da, db; elect.sync _|e, 0xffffffff; setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3}; mov.b64 db, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], da, db, %4, [%6], [%7], p; }"
      ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tmem_copy_scales(uint32_t taddr, uint32_t lo, uint32_t hi) {
  asm volatile("{ .reg .pred e; .reg .b64 d; elect.sync _|e, 0xffffffff; mov.b64 d, {%1, %2};\n\t"
               "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], d; }" ::"r"(taddr), "r"(lo), "r"(hi)
               : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "{ .reg .pred e; elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0]; }" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive fp32 accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void sts128_u32(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 lds128_u32(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void record_error(int32_t* err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

template <typename OutT, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
mxfp8_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                  const __grid_constant__ GemmArgs a) {
  using C = GemmCfg<BN>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kStageBytes = C::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  // operand tiles need 1024-byte alignment (128-byte swizzle atoms)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  // full[s], empty[s], acc_full, acc_empty, tmem slot
  const uint32_t bars = base + kStages * kStageBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
  const uint32_t acc_full = bars + 8u * (2 * kStages);
  const uint32_t acc_empty = acc_full + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kStages * kStageBytes + 8 * (2 * kStages + 2));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // bf16 epilogue staging rows of this warp (epilogue warps only)
  const uint32_t epi = bars + kBarBytes + kEpiStageBytes * uint32_t(warp >= 2 ? warp - 2 : 0);
  const uint32_t n_my = (a.ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;  // grid <= tiles

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(C::kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; s++) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpilogueWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    // stages run on across tiles, so the next tile's loads overlap this
    // tile's last MMAs and its epilogue
    uint32_t it = 0;
    for (uint32_t i = 0; i < n_my; i++) {
      const uint32_t tile = blockIdx.x + i * gridDim.x;
      const uint32_t m_blk = tile / a.n_tiles_n, n_blk = tile % a.n_tiles_n;
      const uint8_t* sfa = a.sfa + (uint64_t(m_blk) * a.kp4) * kSfTile;
      // B's 128-row scale blocks of this tile that exist (the last tile of a
      // ragged N may have fewer than BN / 128; its missing rows are never stored)
      const uint32_t b0 = n_blk * C::kSfbTiles;
      const uint32_t nsfb = min(C::kSfbTiles, a.nb128 - b0);
      const uint32_t tx = C::kTileA + C::kTileB + kSfTile * (1 + nsfb);
      bool ok = true;
      for (uint32_t kb = 0; kb < a.nk; kb++, it++) {
        const int s = it % kStages;
        const uint32_t phase = (it / kStages) & 1u;
        if (!mbar_wait(empty_bar(s), phase ^ 1u, kWaitNs)) {
          record_error(a.err, kErrEmptyWait);
          ok = false;
          break;
        }
        const uint32_t st = base + s * kStageBytes;
        mbar_expect_tx(full_bar(s), tx);
        tma_load_2d(st, &tma_a, full_bar(s), int32_t(kb * kBK), int32_t(m_blk * kBM));
        tma_load_2d(st + C::kTileA, &tma_b, full_bar(s), int32_t(kb * kBK), int32_t(n_blk * BN));
        const uint32_t sf = st + C::kTileA + C::kTileB;
        bulk_load(sf, sfa + uint64_t(kb) * kSfTile, kSfTile, full_bar(s));
        for (uint32_t j = 0; j < nsfb; j++)
          bulk_load(sf + kSfTile * (1 + j), a.sfb + (uint64_t(b0 + j) * a.kp4 + kb) * kSfTile, kSfTile,
                    full_bar(s));
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    // a converged warp with descriptors as 32-bit words plus offsets, as in
    // the pair kernel
    const uint64_t op0 = operand_desc(base);
    const uint64_t sc0 = scale_desc(base + C::kTileA + C::kTileB);
    const uint32_t op_lo = uint32_t(op0), op_hi = uint32_t(op0 >> 32);
    const uint32_t sc_lo = uint32_t(sc0), sc_hi = uint32_t(sc0 >> 32);
    constexpr uint32_t kStageW = kStageBytes >> 4, kTileAW = C::kTileA >> 4, kSfW = kSfTile >> 4;
    uint32_t s = 0, phase = 0;
    for (uint32_t i = 0; i < n_my; i++) {
      // the epilogue must have read the previous tile's accumulator
      if (i > 0 && !__all_sync(0xffffffffu, mbar_wait(acc_empty, (i - 1) & 1u, kWaitNs))) {
        if (lane == 0) record_error(a.err, kErrAccumWait);
        break;
      }
      tc_fence_after();
      bool ok = true;
      for (uint32_t kb = 0; kb < a.nk; kb++) {
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), phase, kWaitNs))) {
          if (lane == 0) record_error(a.err, kErrFullWait);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t so = s * kStageW;
        const uint32_t sfa_t = tmem + BN + C::kSfColsPerStage * s;
        const uint32_t sfb_t = sfa_t + 4u;
        tmem_copy_scales(sfa_t, sc_lo + so, sc_hi);
#pragma unroll
        for (uint32_t j = 0; j < C::kSfbTiles; j++)
          tmem_copy_scales(sfb_t + 4u * j, sc_lo + so + kSfW * (1 + j), sc_hi);
#pragma unroll
        for (uint32_t k = 0; k < 4; k++) {
          mma_mxf8(tmem, op_lo + so + 2 * k, op_lo + so + kTileAW + 2 * k, op_hi, instr_desc<BN>(k),
                   sfa_t | (k << 30), sfb_t | (k << 30), (kb | k) != 0u);
        }
        mma_commit(empty_bar(s));
        if (++s == kStages) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit(acc_full);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // warp w reads accumulator lanes (rows) 32 (w % 4) .. 32 (w % 4) + 31
    const uint32_t quarter = uint32_t(warp & 3);
    const uint32_t taddr = tmem + ((quarter * 32) << 16);
    for (uint32_t i = 0; i < n_my; i++) {
      const uint32_t tile = blockIdx.x + i * gridDim.x;
      const uint32_t m_blk = tile / a.n_tiles_n, n_blk = tile % a.n_tiles_n;
      // the phase completes once for everyone: a lane that saw it lets the warp go
      const bool have = __any_sync(0xffffffffu, mbar_wait(acc_full, i & 1u, kWaitNs));
      if (!have) {
        if (lane == 0) record_error(a.err, kErrAccumWait);
        break;
      }
      tc_fence_after();
      const uint32_t row = m_blk * kBM + quarter * 32 + lane;
      const uint32_t ncols = min(uint32_t(BN), a.N - n_blk * BN);
      if constexpr (sizeof(OutT) == 2) {
        // the whole row of the accumulator into registers as bf16 pairs, the
        // accumulator handed back, then the stores
        uint32_t w[BN / 2];
#pragma unroll
        for (uint32_t c0 = 0; c0 < uint32_t(BN); c0 += 16) {  // 16 columns a load: no spill at BN = 256
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
#pragma unroll
          for (int q = 0; q < 8; q++)
            w[c0 / 2 + q] = cvt_bf16x2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        // 64-column slices through this warp's staging rows, so that each
        // store instruction writes four rows' 128-byte segments
        const uint32_t row0 = m_blk * kBM + quarter * 32;
        const uint32_t rsub = lane >> 3, ch = lane & 7;
#pragma unroll
        for (uint32_t c0 = 0; c0 < uint32_t(BN); c0 += 64) {
#pragma unroll
          for (int q = 0; q < 8; q++)
            sts128_u32(epi + lane * kEpiPitch + 16 * q,
                       make_uint4(w[c0 / 2 + 4 * q], w[c0 / 2 + 4 * q + 1], w[c0 / 2 + 4 * q + 2],
                                  w[c0 / 2 + 4 * q + 3]));
          __syncwarp();
          const uint32_t col = c0 + 8 * ch;  // first of this lane's 8 columns
#pragma unroll
          for (uint32_t i = 0; i < 8; i++) {
            const uint32_t rr = 4 * i + rsub;
            const uint4 v = lds128_u32(epi + rr * kEpiPitch + 16 * ch);
            if (row0 + rr < a.M && col < ncols)
              st_v4(static_cast<OutT*>(a.d) + uint64_t(row0 + rr) * a.N + uint64_t(n_blk) * BN + col, v);
          }
          __syncwarp();
        }
      } else {
        OutT* drow = static_cast<OutT*>(a.d) + uint64_t(row) * a.N + uint64_t(n_blk) * BN;
#pragma unroll 1
        for (uint32_t c0 = 0; c0 < uint32_t(BN); c0 += 32) {
          uint32_t r[32];
          tmem_ld32(taddr + c0, r);  // every lane of the warp takes part
          if (c0 + 32 >= uint32_t(BN)) {
            // the whole accumulator is in registers: hand it back to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          if (row >= a.M || c0 >= ncols) continue;
          if (c0 + 32 <= ncols) {
#pragma unroll
            for (int q = 0; q < 8; q++)
              st_v4(drow + c0 + 4 * q, make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
          } else {
#pragma unroll
            for (uint32_t q = 0; q < 32; q++)
              if (c0 + q < ncols) st_u32(drow + c0 + q, r[q]);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------ CTA-pair kernel
//
// Two CTAs of a cluster (one per SM) share one 256 x 256 output tile through
// the pair form of the block-scaled MMA (tcgen05.mma.cta_group::2, M = 256):
// CTA r of the pair holds A rows 128 r .. 128 r + 127 of the tile and B rows
// 128 r .. 128 r + 127, and the MMA, issued by the even CTA, reads B from
// both. Each CTA therefore loads 32 KiB of operands per K block for the work
// that takes 48 KiB in the single-CTA kernel, and six stages fit. Scales: each
// CTA holds its own A scale tile and both B scale tiles of the pair tile in
// shared memory; the even CTA copies them into both CTAs' tensor memory
// (tcgen05.cp.cta_group::2). Every TMA load of both CTAs completes on the even
// CTA's "full" barrier; the even CTA's commits arrive on the "empty" and
// "acc_full" barriers of both CTAs; both CTAs' epilogue warps arrive on the
// even CTA's "acc_empty". Each CTA's accumulator (its 128 rows x 256 columns)
// is in its own tensor memory and is written out by its own epilogue warps.

constexpr int kPairStages = 6;
constexpr uint32_t kPairTileA = kBM * kBK;                    // 16 KiB: this CTA's A rows
constexpr uint32_t kPairTileB = 128 * kBK;                    // 16 KiB: this CTA's half of B
constexpr uint32_t kPairStageBytes =
    (kPairTileA + kPairTileB + 3 * kSfTile + 1023u) & ~1023u;  // + A scales + both B scale tiles
constexpr uint32_t kPairStageTx = kPairTileA + kPairTileB + 3 * kSfTile;  // one CTA's bytes
constexpr uint32_t kPairSfCols = 12;                          // tensor-memory scale columns a stage
constexpr uint32_t kPairTmemCols = 512;
constexpr uint32_t kPairSmemBytes =
    kPairStages * kPairStageBytes + kBarBytes + kEpiStageBytes * kEpilogueWarps + 1024;
static_assert(256 + kPairStages * kPairSfCols <= kPairTmemCols, "tensor memory");
static_assert(kPairSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on a
// barrier of the pair (given by its shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(x), "r"(y)
      : "memory");
}

// The pair forms of mma_mxf8, tmem_copy_scales and mma_commit, for a
// converged warp: each instruction is issued by the one lane that elect.sync
// picks, inside the same asm block (no branch around it). The commit arrives
// on the barrier at this shared offset in both CTAs of the pair once the
// MMAs issued so far have completed.
__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                              uint32_t hi, uint32_t idesc, uint32_t sfa_tmem,
                                              uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p, e; .reg .b64 da, db; elect.sync _|e, 0xffffffff; setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3}; mov.b64 db, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], da, db, %4, [%6], [%7], p; }"
      ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tmem_copy_scales_pair(uint32_t taddr, uint32_t lo, uint32_t hi) {
  asm volatile("{ .reg .pred e; .reg .b64 d; elect.sync _|e, 0xffffffff; mov.b64 d, {%1, %2};\n\t"
               "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], d; }" ::"r"(taddr), "r"(lo), "r"(hi)
               : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "{ .reg .pred e; elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1; }"
      ::"r"(bar), "h"(uint16_t(3))
      : "memory");
}

// Instruction descriptor as instr_desc<256> but for the pair's M = 256.
__device__ __forceinline__ uint32_t instr_desc_pair(uint32_t k) {
  return (k << 4) | (uint32_t(256 >> 3) << 17) | (1u << 23) | (uint32_t(256 >> 4) << 24) | (k << 29);
}

template <typename OutT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
mxfp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                       const __grid_constant__ CUtensorMap tma_sfa,
                       const __grid_constant__ CUtensorMap tma_sfb, const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bars = base + kPairStages * kPairStageBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (kPairStages + s); };
  const uint32_t acc_full = bars + 8u * (2 * kPairStages);
  const uint32_t acc_empty = acc_full + 8u;
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(smem + kPairStages * kPairStageBytes + 8 * (2 * kPairStages + 2));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t n_my = (a.ntiles - pair + npairs - 1) / npairs;  // npairs <= tiles
  const uint32_t epi = bars + kBarBytes + kEpiStageBytes * uint32_t(warp >= 2 ? warp - 2 : 0);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(kPairTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kPairStages; s++) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpilogueWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    const uint32_t lead_full0 = cluster_addr(full_bar(0), 0);
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t i = 0; i < n_my && ok; i++) {
      const uint32_t tile = pair + i * npairs;
      const uint32_t m_blk = tile / a.n_tiles_n, n_blk = tile % a.n_tiles_n;
      const int32_t a_row = int32_t(m_blk * 256 + 128 * rank);
      const int32_t b_row = int32_t(n_blk * 256 + 128 * rank);
      // rows of 128 bytes in the scale maps: tile (row block, K block) at 4 (rb kp4 + kb)
      const uint32_t sfa_rb = m_blk * 2 + rank, sfb_rb = n_blk * 2;
      for (uint32_t kb = 0; kb < a.nk; kb++, it++) {
        const int s = it % kPairStages;
        const uint32_t phase = (it / kPairStages) & 1u;
        if (!mbar_wait(empty_bar(s), phase ^ 1u, kWaitNs)) {
          record_error(a.err, kErrEmptyWait);
          ok = false;
          break;
        }
        if (rank == 0) mbar_expect_tx(full_bar(s), 2 * kPairStageTx);
        const uint32_t bar = lead_full0 + 8u * s;
        const uint32_t st = base + s * kPairStageBytes;
        tma_load_2d_pair(st, &tma_a, bar, int32_t(kb * kBK), a_row);
        tma_load_2d_pair(st + kPairTileA, &tma_b, bar, int32_t(kb * kBK), b_row);
        const uint32_t sf = st + kPairTileA + kPairTileB;
        tma_load_2d_pair(sf, &tma_sfa, bar, 0, int32_t(4 * (sfa_rb * a.kp4 + kb)));
        tma_load_2d_pair(sf + kSfTile, &tma_sfb, bar, 0, int32_t(4 * (sfb_rb * a.kp4 + kb)));
        tma_load_2d_pair(sf + 2 * kSfTile, &tma_sfb, bar, 0, int32_t(4 * ((sfb_rb + 1) * a.kp4 + kb)));
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------------- MMA issuer
    // The whole warp runs this loop, converged; one elected lane issues each
    // tcgen05 instruction (measured 8 % faster overall than lane 0 running
    // the loop alone with the other lanes parked).
    // Descriptors as 32-bit words: the address field holds addr / 16 of a
    // shared address below 256 KiB, so moving an operand by d bytes (a
    // multiple of 16) adds d / 16 to the low word and leaves the high word.
    // The scalar work sits between the tcgen05 instructions, so it is kept to
    // a few adds (building each descriptor from its address instead, with
    // the ring position as it % 6, measured about 10 % slower overall).
    const uint64_t op0 = operand_desc(base);
    const uint64_t sc0 = scale_desc(base + kPairTileA + kPairTileB);
    const uint32_t op_lo = uint32_t(op0), op_hi = uint32_t(op0 >> 32);
    const uint32_t sc_lo = uint32_t(sc0), sc_hi = uint32_t(sc0 >> 32);
    constexpr uint32_t kStageW = kPairStageBytes >> 4, kTileAW = kPairTileA >> 4, kSfW = kSfTile >> 4;
    uint32_t s = 0, phase = 0;
    for (uint32_t i = 0; i < n_my; i++) {
      if (i > 0 && !__all_sync(0xffffffffu, mbar_wait(acc_empty, (i - 1) & 1u, kWaitNs))) {
        if (lane == 0) record_error(a.err, kErrAccumWait);
        break;
      }
      tc_fence_after();
      bool ok = true;
      for (uint32_t kb = 0; kb < a.nk; kb++) {
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), phase, kWaitNs))) {
          if (lane == 0) record_error(a.err, kErrFullWait);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t so = s * kStageW;
        const uint32_t sfa_t = tmem + 256 + kPairSfCols * s;
        const uint32_t sfb_t = sfa_t + 4u;
        // B's two tiles first: this order measured about 0.6 % faster than
        // A first (alternating rounds, every round)
        tmem_copy_scales_pair(sfb_t, sc_lo + so + kSfW, sc_hi);
        tmem_copy_scales_pair(sfb_t + 4u, sc_lo + so + 2 * kSfW, sc_hi);
        tmem_copy_scales_pair(sfa_t, sc_lo + so, sc_hi);
#pragma unroll
        for (uint32_t k = 0; k < 4; k++) {
          mma_mxf8_pair(tmem, op_lo + so + 2 * k, op_lo + so + kTileAW + 2 * k, op_hi,
                          instr_desc_pair(k), sfa_t | (k << 30), sfb_t | (k << 30), (kb | k) != 0u);
        }
        mma_commit_pair(empty_bar(s));
        if (++s == kPairStages) {
          s = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit_pair(acc_full);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = uint32_t(warp & 3);
    const uint32_t taddr = tmem + ((quarter * 32) << 16);
    const uint32_t lead_acc_empty = cluster_addr(acc_empty, 0);
    for (uint32_t i = 0; i < n_my; i++) {
      const uint32_t tile = pair + i * npairs;
      const uint32_t m_blk = tile / a.n_tiles_n, n_blk = tile % a.n_tiles_n;
      const bool have = __any_sync(0xffffffffu, mbar_wait(acc_full, i & 1u, kWaitNs));
      if (!have) {
        if (lane == 0) record_error(a.err, kErrAccumWait);
        break;
      }
      tc_fence_after();
      const uint32_t row0 = m_blk * 256 + 128 * rank + quarter * 32;
      const uint32_t ncols = min(256u, a.N - n_blk * 256);
      if constexpr (sizeof(OutT) == 2) {
        // 16 columns per tensor-memory load: the whole row (128 bf16 pairs)
        // then fits in registers without spilling
        uint32_t w[128];
#pragma unroll
        for (uint32_t c0 = 0; c0 < 256u; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
#pragma unroll
          for (int q = 0; q < 8; q++)
            w[c0 / 2 + q] = cvt_bf16x2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(lead_acc_empty);
        const uint32_t rsub = lane >> 3, ch = lane & 7;
#pragma unroll
        for (uint32_t c0 = 0; c0 < 256u; c0 += 64) {
#pragma unroll
          for (int q = 0; q < 8; q++)
            sts128_u32(epi + lane * kEpiPitch + 16 * q,
                       make_uint4(w[c0 / 2 + 4 * q], w[c0 / 2 + 4 * q + 1], w[c0 / 2 + 4 * q + 2],
                                  w[c0 / 2 + 4 * q + 3]));
          __syncwarp();
          const uint32_t col = c0 + 8 * ch;
#pragma unroll
          for (uint32_t j = 0; j < 8; j++) {
            const uint32_t rr = 4 * j + rsub;
            const uint4 v = lds128_u32(epi + rr * kEpiPitch + 16 * ch);
            if (row0 + rr < a.M && col < ncols)
              st_v4(static_cast<OutT*>(a.d) + uint64_t(row0 + rr) * a.N + uint64_t(n_blk) * 256 + col, v);
          }
          __syncwarp();
        }
      } else {
        const uint32_t row = row0 + lane;
        OutT* drow = static_cast<OutT*>(a.d) + uint64_t(row) * a.N + uint64_t(n_blk) * 256;
#pragma unroll 1
        for (uint32_t c0 = 0; c0 < 256u; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(taddr + c0, r);
          if (c0 + 32 >= 256u) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead_acc_empty);
          }
          if (row >= a.M || c0 >= ncols) continue;
          if (c0 + 32 <= ncols) {
#pragma unroll
            for (int q = 0; q < 8; q++)
              st_v4(drow + c0 + 4 * q, make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
          } else {
#pragma unroll
            for (uint32_t q = 0; q < 32; q++)
              if (c0 + q < ncols) st_u32(drow + c0 + q, r[q]);
          }
        }
      }
    }
  }

  // neither CTA leaves while the other may still reach its shared memory or
  // tensor memory (barrier arrivals, MMA operand reads, scale copies)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPairTmemCols)
                 : "memory");
  }
}

// The GEMM's bounded wait, both ways (see mxq_check_bounded_wait): a barrier
// that nothing arrives on must make mbar_wait give up after timeout_ns, and
// one whose phase has completed must let it return at once. One thread; no
// asynchronous operation refers to either barrier, so the CTA may exit with
// the first one's phase still open.
__global__ void bounded_wait_check_kernel(uint64_t timeout_ns, int64_t* result) {
  __shared__ alignas(8) uint64_t bars[2];
  if (threadIdx.x != 0) return;
  const uint32_t never = smem_u32(&bars[0]), done = smem_u32(&bars[1]);
  mbar_init(never, 1);
  mbar_init(done, 1);
  const uint64_t t0 = globaltimer();
  const bool first = mbar_wait(never, 0, timeout_ns);
  const uint64_t t1 = globaltimer();
  mbar_arrive(done);
  const bool second = mbar_wait(done, 0, timeout_ns);
  result[0] = first ? 0 : 1;
  result[1] = second ? 1 : 0;
  result[2] = int64_t(t1 - t0);
  result[3] = 0;
}

// ------------------------------------------------------------------ host

// [rows, K] bytes, row stride K, boxes of box_rows rows x 128 bytes,
// 128-byte swizzle; out-of-range rows and columns read as zero.
bool make_operand_map(CUtensorMap* map, const uint8_t* p, uint64_t rows, uint64_t K,
                      uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K};
  const cuuint32_t box[2] = {uint32_t(kBK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A swizzled scale array seen as rows of 128 bytes; one load takes a 512-byte
// 128 x 4 scale tile (4 rows), no swizzle.
bool make_scale_map(CUtensorMap* map, const uint8_t* p, uint64_t bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {128, bytes / 128};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, 4};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two that can be resident at once on the current device (at
// least one), for the CTA-pair kernel's persistent grid.
template <typename OutT>
uint32_t max_pair_clusters() {
  static std::atomic<int> cached[256];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return uint32_t(n);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 256);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int c = 0;
  if (cudaOccupancyMaxActiveClusters(&c, mxfp8_gemm_pair_kernel<OutT>, &cfg) != cudaSuccess || c <= 0) {
    (void)cudaGetLastError();
    c = sm_count() / 2;
  }
  cached[dev].store(c, std::memory_order_relaxed);
  return uint32_t(c);
}

template <typename OutT>
mxq_status launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                            const CUtensorMap& tsb, const GemmArgs& args, cudaStream_t s) {
  const cudaError_t attr_err = ensure_smem_limit<mxfp8_gemm_pair_kernel<OutT>>(int(kPairSmemBytes));
  if (attr_err != cudaSuccess) {
    record_cuda_error(attr_err);
    return MXQ_ERR_CUDA;
  }
  GemmArgs a2 = args;
  a2.n_tiles_n = (args.N + 255) / 256;
  a2.ntiles = a2.n_tiles_n * ((args.M + 255) / 256);
  const uint32_t clusters = max_pair_clusters<OutT>();
  const uint32_t pairs = a2.ntiles < clusters ? a2.ntiles : clusters;
  mxfp8_gemm_pair_kernel<OutT><<<2 * pairs, kGemmThreads, kPairSmemBytes, s>>>(ta, tb, tsa, tsb, a2);
  return check_launch();
}

template <typename OutT, int BN>
mxq_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args,
                       cudaStream_t s) {
  constexpr uint32_t kSmemBytes = GemmCfg<BN>::kSmemBytes;
  const cudaError_t attr_err = ensure_smem_limit<mxfp8_gemm_kernel<OutT, BN>>(int(kSmemBytes));
  if (attr_err != cudaSuccess) {
    record_cuda_error(attr_err);
    return MXQ_ERR_CUDA;
  }
  GemmArgs a2 = args;
  a2.n_tiles_n = (args.N + BN - 1) / BN;
  a2.ntiles = a2.n_tiles_n * ((args.M + kBM - 1) / kBM);
  const uint32_t sms = uint32_t(sm_count());
  const uint32_t grid = a2.ntiles < sms ? a2.ntiles : sms;
  mxfp8_gemm_kernel<OutT, BN><<<grid, kGemmThreads, kSmemBytes, s>>>(ta, tb, a2);
  return check_launch();
}

}  // namespace
}  // namespace mxq

extern "C" mxq_status mxfp8_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb,
                                 const uint8_t* sb_swz, int64_t M, int64_t N, int64_t K, void* d,
                                 int out_dt, int32_t* error_flag, mxq_stream_t stream) {
  using namespace mxq;
  if (!valid_dtype(out_dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || K < 0 || K % 32 != 0 || N % 16 != 0) return MXQ_ERR_SHAPE;
  if (M > 0x7fffff80ll || N > 0x7fffff80ll || K > 0x7fffff80ll) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!d) return MXQ_ERR_NULL;
  if (!aligned16(d)) return MXQ_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    const cudaError_t e = cudaMemsetAsync(d, 0, size_t(M) * size_t(N) * elem_size(out_dt), s);
    if (e != cudaSuccess) {
      record_cuda_error(e);
      return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
  }
  if (!qa || !qb || !sa_swz || !sb_swz) return MXQ_ERR_NULL;
  if (!aligned16(qa) || !aligned16(qb) || !aligned16(sa_swz) || !aligned16(sb_swz))
    return MXQ_ERR_ALIGN;
  // 256 x 256 tiles over a CTA pair when both sides exceed one 128-row
  // block; otherwise one CTA per tile, 128 x 256 (128 x 128 when N <= 128)
  const bool wide = N > 128;
  const bool paired = wide && M > 128;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_operand_map(&ta, qa, uint64_t(M), uint64_t(K), kBM) ||
      !make_operand_map(&tb, qb, uint64_t(N), uint64_t(K), (wide && !paired) ? 256u : 128u))
    return MXQ_ERR_CUDA;
  GemmArgs args{};
  args.sfa = sa_swz;
  args.sfb = sb_swz;
  args.d = d;
  args.err = error_flag;
  args.M = uint32_t(M);
  args.N = uint32_t(N);
  args.nk = uint32_t((K + kBK - 1) / kBK);
  args.kp4 = args.nk;
  args.nb128 = uint32_t((N + 127) / 128);
  if (paired) {
    const uint64_t sa_bytes = (uint64_t(M) + 127) / 128 * args.kp4 * kSfTile;
    const uint64_t sb_bytes = (uint64_t(N) + 127) / 128 * args.kp4 * kSfTile;
    if (!make_scale_map(&tsa, sa_swz, sa_bytes) || !make_scale_map(&tsb, sb_swz, sb_bytes))
      return MXQ_ERR_CUDA;
    return out_dt == MXQ_BF16 ? launch_gemm_pair<uint16_t>(ta, tb, tsa, tsb, args, s)
                              : launch_gemm_pair<float>(ta, tb, tsa, tsb, args, s);
  }
  if (out_dt == MXQ_BF16)
    return wide ? launch_gemm<uint16_t, 256>(ta, tb, args, s) : launch_gemm<uint16_t, 128>(ta, tb, args, s);
  return wide ? launch_gemm<float, 256>(ta, tb, args, s) : launch_gemm<float, 128>(ta, tb, args, s);
}

extern "C" mxq_status mxq_check_bounded_wait(int64_t timeout_ns, int64_t* result,
                                             mxq_stream_t stream) {
  using namespace mxq;
  if (timeout_ns < 1000 || timeout_ns > 1000000000) return MXQ_ERR_ARG;
  if (!result) return MXQ_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(result) & 7u) return MXQ_ERR_ALIGN;
  bounded_wait_check_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      uint64_t(timeout_ns), result);
  return launched(cudaGetLastError());
}
