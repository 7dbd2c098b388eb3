// colwise.cu -- MXFP8 columnwise quantize (groups of 32 consecutive rows of
// one column, the operand layout of a backward GEMM), optionally fused with
// the rowwise quantize so that the input is read once, for sm_100a.
//
// Method: each column group is quantized by the rowwise rule of mx_rowwise.cu
// (NaN-ignoring amax, E8M0 byte = 127 / 254 / clamp(E(amax) - 8, 0, 254),
// E4M3 RNE with saturation). Following the adapter contract of "PR #1935
// 完整报告 -- Use TransformerEngine for MXFP8 quantization" (实现拆解 item 1:
// zero-pad rows to a multiple of 32, quantize, crop back), rows past M count
// as zeros in the last group of each column; for columnwise groups that
// padding is part of the result. Outputs are transposed and cropped:
// q_t [N, M] (q_t[c, r] is the code of x[r, c]) and scale_t [N, ceil(M/32)].
//
// Work split (HBM-bound: 2 bytes read, 1 + 1/32 written per bf16 element;
// the fused mode writes 2 + 2/32): persistent CTAs (two per multiprocessor)
// walk tiles of 128 rows x 256 bytes (128 bf16 or 64 fp32 columns). A tile is
// staged in shared memory with 16-byte cp.async copies (rows past M and
// columns past N zero-filled) into one of two buffers while the previous tile
// is worked on, so loads overlap compute and stores; row pitch 272 bytes so
// that both phases below read shared memory without bank conflicts.
//  - Column phase: a thread owns one 4-byte word column (two bf16 columns or
//    one fp32 column) and one 32-row group, reads its 32 words down the
//    rows (consecutive lanes read consecutive words), reduces both bf16
//    column maxima with one max.xorsign.abs.bf16x2 tree, and writes a 32-byte
//    column group of q_t per column (a full 32-byte sector).
//  - Row phase (fused mode): a thread owns one (row, 32-column) group of the
//    tile, reads it as 16-byte shared loads and writes 32 bytes of q.
// The transposed codes are staged in shared memory as well, so that every
// q_t row segment of the tile (128 bytes) is written as a full line by 8
// consecutive lanes, and the tile's 4 scale bytes of a column as one word.
#include "common.cuh"

namespace mxq {
namespace {

constexpr int kTileRows = 128;
constexpr int kRowBytes = 256;               // one tile row
constexpr int kPitch = kRowBytes + 16;       // padded shared-memory row pitch
constexpr int kWordCols = kRowBytes / 4;     // 64 word columns per tile
constexpr int kOutPitch = kTileRows + 16;    // shared pitch of a transposed code row
constexpr uint32_t kInBytes = kTileRows * kPitch;           // one staged input tile
constexpr uint32_t kQsBytes = (kRowBytes / 2) * kOutPitch;  // transposed codes (bf16: 128 columns)
constexpr uint32_t kSsBytes = (kRowBytes / 2) * 4;           // column scales of a tile
constexpr int kRowPitch = kRowBytes / 2 + 16;                // shared pitch of a row of codes
constexpr uint32_t kQrBytes = kTileRows * kRowPitch;          // rowwise codes (fused mode)
constexpr uint32_t kSrBytes = kTileRows * 4;                  // rowwise scales (fused mode)
constexpr uint32_t kColSmem = 2 * kInBytes + kQsBytes + kSsBytes;
constexpr uint32_t kFusedSmem = kColSmem + kQrBytes + kSrBytes;

// 16-byte asynchronous copy global -> shared; src_bytes == 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
  return v;
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
  return v;
}

__device__ __forceinline__ void sts128(uint8_t* p, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(p))),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

struct ColArgs {
  const uint8_t* x;      // input base (bytes)
  int64_t ld_bytes;      // input row stride in bytes
  int64_t M, N;
  uint32_t n_ct;         // column tiles
  uint32_t ntiles;       // row tiles x column tiles
  uint32_t gt;           // groups per column: ceil(M / 32)
  uint8_t* q_t;          // [N, M]
  uint8_t* scale_t;      // [N, gt]
  uint8_t* q;            // [M, N] (fused mode)
  uint8_t* scale;        // [M, N / 32] (fused mode)
  bool q_t_aligned;      // every q_t row start is 16-byte aligned (M % 16 == 0)
  bool scale_words;      // scale_t 4-byte aligned and ceil(M/32) % 4 == 0
  bool row_scale_words;  // fused mode: scale 4-byte aligned and (N / 32) % 4 == 0
};

// max.xorsign.abs over N bf16 pairs as a pairwise tree (depth log2 N rather
// than a chain of N - 1 dependent maxima); the result's sign bits are junk.
template <int N>
__device__ __forceinline__ uint32_t absmax_tree(const uint32_t (&v)[N]) {
  uint32_t m[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; i++) m[i] = absmax_bf16x2(v[2 * i], v[2 * i + 1]);
#pragma unroll
  for (int n = N / 4; n >= 1; n /= 2) {
#pragma unroll
    for (int i = 0; i < n; i++) m[i] = absmax_bf16x2(m[2 * i], m[2 * i + 1]);
  }
  return m[0];
}

// Sixteen code pairs (first code in the low byte) as two 16-byte halves.
__device__ __forceinline__ void pack_codes(const uint32_t (&c)[16], uint4& lo, uint4& hi) {
  lo = make_uint4(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410),
                  __byte_perm(c[4], c[5], 0x5410), __byte_perm(c[6], c[7], 0x5410));
  hi = make_uint4(__byte_perm(c[8], c[9], 0x5410), __byte_perm(c[10], c[11], 0x5410),
                  __byte_perm(c[12], c[13], 0x5410), __byte_perm(c[14], c[15], 0x5410));
}

// 32 E4M3 codes of 32 fp32 values times the power-of-two multiplier `mul`.
__device__ __forceinline__ void column_codes(const float (&f)[32], float mul, uint4& lo, uint4& hi) {
  uint32_t c[16];
#pragma unroll
  for (int k = 0; k < 16; k++) {
    const float2 p = mul2(f[2 * k], f[2 * k + 1], mul);
    c[k] = cvt_e4m3x2(p.x, p.y);
  }
  pack_codes(c, lo, hi);
}

// 32 E4M3 codes of 32 consecutive bf16 elements of a row (16 packed words)
// times the power of two `mul`.
__device__ __forceinline__ void row_codes_bf16(const uint32_t (&w)[16], float mul, uint4& lo, uint4& hi) {
  uint32_t c[16];
#pragma unroll
  for (int k = 0; k < 16; k++) {
    const float2 p = mul_bf16x2_pow2(w[k], mul);
    c[k] = cvt_e4m3x2(p.x, p.y);
  }
  pack_codes(c, lo, hi);
}

// 32 E4M3 codes of one bf16 column: half H of the words v[0..31] (one word
// per row) times the power of two `mul`.
template <int H>
__device__ __forceinline__ void column_codes_bf16(const uint32_t (&v)[32], float mul, uint4& lo, uint4& hi) {
  uint32_t c[16];
#pragma unroll
  for (int k = 0; k < 16; k++) {
    const float2 p = mul_bf16_pow2<H, H>(v[2 * k], v[2 * k + 1], mul);
    c[k] = cvt_e4m3x2(p.x, p.y);
  }
  pack_codes(c, lo, hi);
}

template <typename InT, bool ROW>
__global__ void __launch_bounds__(kThreads, 2)
mxfp8_colwise_kernel(const __grid_constant__ ColArgs a) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kEsize = sizeof(InT);
  constexpr int kTileCols = kRowBytes / kEsize;
  uint8_t* const qs = smem + 2 * kInBytes;  // transposed codes [column][row]
  uint8_t* const ss = qs + kQsBytes;        // scales [column][group]
  uint8_t* const qr = ss + kSsBytes;        // fused mode: rowwise codes [row][column]
  uint8_t* const sr = qr + kQrBytes;        // fused mode: rowwise scales [row][group]
  const int t = threadIdx.x;

  // stages tile `tile` into input buffer `b`: 128 rows x 16 chunks of 16
  // bytes, 8 chunks per thread, zeros past M and N
  auto stage = [&](uint32_t tile, int b) {
    const uint32_t ct = tile % a.n_ct, rt = tile / a.n_ct;
    const int64_t r0 = int64_t(rt) * kTileRows, c0 = int64_t(ct) * kTileCols;
    const int rows = a.M - r0 < kTileRows ? int(a.M - r0) : kTileRows;
    const int row_bytes = (a.N - c0 < kTileCols ? int(a.N - c0) : kTileCols) * kEsize;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(smem + b * kInBytes));
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int idx = i * kThreads + t, r = idx >> 4, ch = idx & 15;
      const bool ok = r < rows && ch * 16 < row_bytes;
      const uint8_t* src = ok ? a.x + (r0 + r) * a.ld_bytes + c0 * kEsize + ch * 16 : a.x;
      cp_async16(dst + r * kPitch + ch * 16, src, ok ? 16u : 0u);
    }
  };

  int b = 0;
  if (blockIdx.x < a.ntiles) stage(blockIdx.x, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (uint32_t tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x, b ^= 1) {
    // the next tile's copies go out before this one is worked on
    if (tile + gridDim.x < a.ntiles) stage(tile + gridDim.x, b ^ 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();  // this tile is in shared memory; the previous one's outputs are written

    const uint8_t* in = smem + b * kInBytes;
    const uint32_t ct = tile % a.n_ct, rt = tile / a.n_ct;
    const int64_t r0 = int64_t(rt) * kTileRows, c0 = int64_t(ct) * kTileCols;
    const int rows = a.M - r0 < kTileRows ? int(a.M - r0) : kTileRows;
    const int row_bytes = (a.N - c0 < kTileCols ? int(a.N - c0) : kTileCols) * kEsize;  // multiple of 32
    // row phase (fused mode): (row, 32-column group) pairs of the tile
    if constexpr (ROW) {
      constexpr int kGroups = kTileCols / 32;             // 4 (bf16) or 2 (fp32)
      constexpr int kPerThread = kTileRows * kGroups / kThreads;
#pragma unroll
      for (int j = 0; j < kPerThread; j++) {
        const int r = t & (kTileRows - 1);
        const int k = (t >> 7) * kPerThread + j;
        if (r < rows && k * 32 * kEsize < row_bytes) {
          const uint8_t* src = in + r * kPitch + k * 32 * kEsize;
          uint32_t b;
          uint4 lo, hi;
          if constexpr (kEsize == 2) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 4; i++) {
              const uint4 q4 = lds128(src + 16 * i);
              w[4 * i] = q4.x; w[4 * i + 1] = q4.y; w[4 * i + 2] = q4.z; w[4 * i + 3] = q4.w;
            }
            const uint32_t m = absmax_tree(w) & 0x7fff7fffu;
            b = mx_scale_byte<8>(fmaxf(fmaxf(bf16_lo(m), bf16_hi(m)), 0.0f));
            row_codes_bf16(w, pow2_quant(b), lo, hi);
          } else {
            float f[32];
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const uint4 q4 = lds128(src + 16 * i);
              f[4 * i] = __uint_as_float(q4.x); f[4 * i + 1] = __uint_as_float(q4.y);
              f[4 * i + 2] = __uint_as_float(q4.z); f[4 * i + 3] = __uint_as_float(q4.w);
            }
#pragma unroll
            for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(f[i]));
            b = mx_scale_byte<8>(amax);
            column_codes(f, pow2_quant(b), lo, hi);
          }
          sts128(qr + r * kRowPitch + 32 * k, lo);
          sts128(qr + r * kRowPitch + 32 * k + 16, hi);
          sr[4 * r + k] = uint8_t(b);
        }
      }
    }
    // column phase: word column w, group g (rows 32g .. 32g + 31 of the tile);
    // the codes go to the transposed tile qs[column][row].
    {
      const int w = t & (kWordCols - 1), g = t >> 6;
      const bool active = 32 * g < rows && w * 4 < row_bytes;
      uint4 code[kEsize == 2 ? 4 : 2];
      uint32_t sb[2] = {0, 0};
      if (active) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; i++) v[i] = lds32(in + (32 * g + i) * kPitch + 4 * w);
        if constexpr (kEsize == 2) {
          const uint32_t m = absmax_tree(v) & 0x7fff7fffu;
          sb[0] = mx_scale_byte<8>(fmaxf(bf16_lo(m), 0.0f));
          sb[1] = mx_scale_byte<8>(fmaxf(bf16_hi(m), 0.0f));
          column_codes_bf16<0>(v, pow2_quant(sb[0]), code[0], code[1]);
          column_codes_bf16<1>(v, pow2_quant(sb[1]), code[2], code[3]);
        } else {
          float f[32];
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; i++) {
            f[i] = __uint_as_float(v[i]);
            amax = fmaxf(amax, fabsf(f[i]));
          }
          sb[0] = mx_scale_byte<8>(amax);
          column_codes(f, pow2_quant(sb[0]), code[0], code[1]);
        }
      }
      if (active) {
        constexpr int kCols = 4 / kEsize;  // columns per word
#pragma unroll
        for (int e = 0; e < kCols; e++) {
          const int col = kCols * w + e;
          sts128(qs + col * kOutPitch + 32 * g, code[2 * e]);
          sts128(qs + col * kOutPitch + 32 * g + 16, code[2 * e + 1]);
          ss[col * 4 + g] = uint8_t(sb[e]);
        }
      }
    }
    __syncthreads();

    // write the transposed tile: 8 consecutive lanes write one q_t row's
    // 128-byte segment (rows of the tile past M are not written)
    {
      const int cols = row_bytes / kEsize;
#pragma unroll
      for (int i = 0; i < kTileCols * 8 / kThreads; i++) {
        const int idx = i * kThreads + t, col = idx >> 3, ch = idx & 7;
        const int nbytes = rows - 16 * ch;  // valid bytes of this 16-byte chunk
        if (col < cols && nbytes > 0) {
          uint8_t* dst = a.q_t + (c0 + col) * a.M + r0 + 16 * ch;
          const uint4 val = lds128(qs + col * kOutPitch + 16 * ch);
          if (a.q_t_aligned && nbytes >= 16) {
            st_v4(dst, val);
          } else {
            const uint32_t wv[4] = {val.x, val.y, val.z, val.w};
            for (int j = 0; j < (nbytes < 16 ? nbytes : 16); j++)
              st_u8(dst + j, (wv[j >> 2] >> (8 * (j & 3))) & 0xffu);
          }
        }
      }
      // scales: the tile's 4 groups of a column are 4 consecutive bytes of scale_t
      if (t < cols) {
        const int ng = (rows + 31) / 32;
        uint8_t* dst = a.scale_t + (c0 + t) * a.gt + r0 / 32;
        if (ng == 4 && a.scale_words) {
          st_u32(dst, *reinterpret_cast<const uint32_t*>(ss + 4 * t));
        } else {
          for (int j = 0; j < ng; j++) st_u8(dst + j, ss[4 * t + j]);
        }
      }
    }
    // fused mode: the rowwise codes of the tile, one row's segment (128 or 64
    // bytes) written by 8 or 4 consecutive lanes, and its scale bytes
    if constexpr (ROW) {
      constexpr int kChunks = kTileCols / 16;  // 16-byte chunks of a row's codes
      const int64_t S = a.N / 32;
#pragma unroll
      for (int i = 0; i < kTileRows * kChunks / kThreads; i++) {
        const int idx = i * kThreads + t, r = idx / kChunks, ch = idx % kChunks;
        if (r < rows && ch * 16 < row_bytes / kEsize)
          st_v4(a.q + (r0 + r) * a.N + c0 + 16 * ch, lds128(qr + r * kRowPitch + 16 * ch));
      }
      if (t < rows) {
        constexpr int kGroups = kTileCols / 32;  // 4 (bf16) or 2 (fp32)
        const int ng = row_bytes / kEsize / 32;
        uint8_t* dst = a.scale + (r0 + t) * S + c0 / 32;
        if (kGroups == 4 && ng == 4 && a.row_scale_words) {
          st_u32(dst, *reinterpret_cast<const uint32_t*>(sr + 4 * t));
        } else {
          for (int j = 0; j < ng; j++) st_u8(dst + j, sr[4 * t + j]);
        }
      }
    }
  }
}

template <typename InT, bool ROW>
mxq_status launch_colwise(const ColArgs& a, uint32_t grid, cudaStream_t s) {
  constexpr uint32_t kSmem = ROW ? kFusedSmem : kColSmem;
  const cudaError_t attr_err = ensure_smem_limit<mxfp8_colwise_kernel<InT, ROW>>(int(kSmem));
  if (attr_err != cudaSuccess) {
    record_cuda_error(attr_err);
    return MXQ_ERR_CUDA;
  }
  return launched(launch_pdl_ex(mxfp8_colwise_kernel<InT, ROW>, grid, kThreads, kSmem, s, a));
}

}  // namespace
}  // namespace mxq

extern "C" mxq_status mxfp8_quantize_columnwise(const void* x, int dt, int64_t M, int64_t N,
                                                int64_t ld_x, uint8_t* qweight_t,
                                                uint8_t* scale_t, uint8_t* qweight,
                                                uint8_t* scale, mxq_stream_t stream) {
  using namespace mxq;
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  const bool fused = qweight != nullptr || scale != nullptr;
  if (M < 0 || N < 0 || N % 16 != 0 || ld_x < N || (fused && N % 32 != 0)) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x || !qweight_t || !scale_t || (fused && (!qweight || !scale))) return MXQ_ERR_NULL;
  const int es = elem_size(dt);
  if (!aligned16(x) || (uint64_t(ld_x) * es) % 16 != 0 || !aligned16(qweight_t) ||
      (fused && !aligned16(qweight)))
    return MXQ_ERR_ALIGN;
  const uint64_t tile_cols = uint64_t(kRowBytes / es);
  const uint64_t tile_rows = kTileRows;
  const uint64_t n_rt = (uint64_t(M) + tile_rows - 1) / tile_rows;
  const uint64_t n_ct = (uint64_t(N) + tile_cols - 1) / tile_cols;
  if (n_rt * n_ct > 0x7fffffffull) return MXQ_ERR_SHAPE;
  ColArgs a{};
  a.x = static_cast<const uint8_t*>(x);
  a.ld_bytes = ld_x * es;
  a.M = M;
  a.N = N;
  a.n_ct = uint32_t(n_ct);
  a.ntiles = uint32_t(n_rt * n_ct);
  a.gt = uint32_t((uint64_t(M) + 31) / 32);
  a.q_t = qweight_t;
  a.scale_t = scale_t;
  a.q = qweight;
  a.scale = scale;
  a.q_t_aligned = (M % 16) == 0;
  a.scale_words = (reinterpret_cast<uintptr_t>(scale_t) & 3u) == 0 && (a.gt & 3u) == 0;
  a.row_scale_words = (reinterpret_cast<uintptr_t>(scale) & 3u) == 0 && ((N / 32) & 3) == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint64_t resident = uint64_t(sm_count()) * 2;
  const uint32_t grid = uint32_t(a.ntiles < resident ? a.ntiles : resident);
  if (dt == MXQ_BF16)
    return fused ? launch_colwise<uint16_t, true>(a, grid, s) : launch_colwise<uint16_t, false>(a, grid, s);
  return fused ? launch_colwise<float, true>(a, grid, s) : launch_colwise<float, false>(a, grid, s);
}
