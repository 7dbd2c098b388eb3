// mx_rowwise.cu -- MX rowwise quantize (compact + optional swizzled scales,
// single tensor or a group of expert tensors in one launch), dequantize and
// fused fake-quantize, for the two MX element formats: MXFP8 (E4M3 codes, one
// byte each) and MXFP4 (E2M1 codes, two per byte), for sm_100a.
//
// Method ("PR #1935 完整报告 -- Use TransformerEngine for MXFP8 quantization",
// 实现拆解 items 1 and 4; "V4 mxfp4 #1372", description and
// mxfp4_simulate_qat): groups of 32 consecutive elements along the last dim;
// per group amax = max |x| over its non-NaN elements, E8M0 byte = 127 for
// amax == 0, 254 for amax == inf, else clamp(E(amax) - emax, 0, 254) where E
// is the biased fp32 exponent field (the same number as floor(log2 amax) +
// 127 - emax, clamped; emax = 8 for E4M3, 2 for E2M1), and
// q = CODE(x * 2^(127 - byte)) rounded to nearest even with saturation to the
// format's largest value (448 for E4M3, 6 for E2M1). Fake-quantize writes
// decode(q) * 2^(byte - 127), the dequantization of the quantization, without
// storing q.
//
// Exactness of the fp32 path: for finite amax the byte is at most 254 - emax,
// so the multiplier 2^(127 - byte) is a normal fp32 power of two and
// x * multiplier is exact whenever the product is an fp32 normal. Products
// below 2^-126 (where fp32 would round) are far below half the smallest
// non-zero code (2^-10 for E4M3, 0.25 for E2M1), so they encode to a zero of
// the right sign either way. An infinite amax gives byte 254 and the
// subnormal multiplier 2^-127 (built from its bit pattern), again exact for
// every product that can encode to non-zero. cvt.rn.satfinite.e4m3x2.f32
// rounds to nearest even, saturates finite and infinite values to +-448,
// keeps the sign of zero and writes every NaN as 0x7F;
// cvt.rn.satfinite.e2m1x2.f32 does the same with +-6 and writes NaN as +6
// (0x7). Both are checked exhaustively against the oracle by the GPU tests.
//
// Work split (HBM-bound: 2 bytes read and 1 + 1/32 (MXFP8) or 1/2 + 1/32
// (MXFP4) written per bf16 element): a lane owns 16 consecutive elements
// (one 256-bit load of bf16, two of fp32, when 32-byte aligned), two lanes a
// group, a warp 16 consecutive groups per step (1 KiB of contiguous bf16) and
// kSteps steps, a CTA kGroupsPerTile consecutive groups. All loads of a lane
// are issued before any is used. The tile's base pointers are formed once in
// 64-bit arithmetic; lane offsets inside a tile are 32-bit, and full tiles
// skip the bounds checks. Rows are never padded: groups do not cross rows,
// so the result for M rows equals the pad-to-32-rows-then-crop contract.
#include "common.cuh"

namespace mxq {
namespace {

constexpr int kGroupsPerStep = 16;  // per warp and step
constexpr int kSteps = 2;
constexpr int kGroupsPerWarp = kGroupsPerStep * kSteps;
constexpr int kGroupsPerTile = kGroupsPerWarp * (kThreads / 32);

// Element formats. kE4M3: MXFP8, one code byte per element. kE2M1: MXFP4, two
// codes per byte, element 2k in the low nibble.
constexpr int kE4M3 = 0;
constexpr int kE2M1 = 1;
template <int FMT>
constexpr int kEmax = FMT == kE4M3 ? 8 : 2;
template <int FMT>
constexpr uint32_t kCodeBytes = FMT == kE4M3 ? 32 : 16;  // code bytes per group

// Byte offset of scale (r, c) in the 128x4-tile layout of block-scaled MMA.
__device__ __forceinline__ uint64_t swz_offset(uint64_t r, uint32_t c, uint32_t Sp4) {
  return (((r >> 7) * Sp4 + (c >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
}

// E4M3 codes of the lane's 16 elements times `mul` (low byte = first element).
template <typename InT>
__device__ __forceinline__ uint4 to_e4m3(const In16<InT>& v, float mul) {
  uint32_t c[8];
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const float2 p = v.scaled(k, mul);
    c[k] = cvt_e4m3x2(p.x, p.y);
  }
  return make_uint4(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410),
                    __byte_perm(c[4], c[5], 0x5410), __byte_perm(c[6], c[7], 0x5410));
}

// E2M1 codes of the lane's 16 elements times `mul`, two per byte with the
// even element in the low nibble (8 bytes, first element in the low byte).
template <typename InT>
__device__ __forceinline__ uint2 to_e2m1(const In16<InT>& v, float mul) {
  uint32_t c[8];
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const float2 p = v.scaled(k, mul);
    c[k] = cvt_e2m1x2(p.x, p.y);
  }
  return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24),
                    c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

template <int MAXE>
struct QuantArgs {
  uint8_t* q;
  uint8_t* scale;
  uint8_t* swz;          // swizzled scales (SWZ only)
  int64_t ld;            // input row stride in elements (STRIDED only)
  FastDiv rows;          // group index -> row, i.e. division by S
  uint32_t S;            // groups per row
  uint32_t Sp4;          // ceil(S / 4)
  uint64_t M;            // rows (SWZ padding)
  uint64_t pad_a;        // swizzle padding entries right of the real scale columns
  uint64_t pad_b;        // swizzle padding entries below the real rows
  int32_t E;             // experts
  const void* x[MAXE];
  uint64_t gbase[MAXE + 1];  // first output group of expert e; gbase[E] = all groups
  uint32_t tbase[MAXE + 1];  // first CTA of expert e; tbase[E] = grid size
};

// Swizzled-scale modes of mx_quant_kernel: none, or one 128x4-tile layout for
// the whole [M, S] scale.
constexpr int kSwzNone = 0;
constexpr int kSwzTensor = 1;

// Row offsets of a stacked tensor's experts in shared memory: off[e] = the
// device offsets clamped into a non-decreasing sequence from off[0] = 0 to
// off[E] = M (so no write can leave the layout, whatever the offsets hold),
// and pb[e] = first row of expert e in the per-expert padded layout,
// pb[e + 1] = pb[e] + ceil((off[e + 1] - off[e]) / 128) * 128. All threads
// load the offsets (one global round trip), then one warp scans them in
// shared memory, 32 entries at a time.
__device__ __forceinline__ void load_expert_rows(const int64_t* __restrict__ g_off, int E,
                                              int64_t M, int64_t* off, int64_t* pb) {
  for (int e = threadIdx.x; e <= E; e += kThreads) {
    int64_t v = e == 0 ? 0 : (e == E ? M : g_off[e]);
    off[e] = v < 0 ? 0 : (v > M ? M : v);
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int64_t carry_off = 0, carry_pb = 0;
    for (int base = 0; base <= E; base += 32) {
      const int e = base + lane;
      int64_t v = e <= E ? off[e] : M;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v = t > v ? t : v;
      }
      v = carry_off > v ? carry_off : v;
      int64_t prev = __shfl_up_sync(kFull, v, 1);
      if (lane == 0) prev = carry_off;
      int64_t d = (e == 0 || e > E) ? 0 : ((v - prev + 127) & ~int64_t(127));
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t t = __shfl_up_sync(kFull, d, o);
        if (lane >= o) d += t;
      }
      d += carry_pb;
      if (e <= E) {
        off[e] = v;
        pb[e] = d;
      }
      carry_off = __shfl_sync(kFull, v, 31);
      carry_pb = __shfl_sync(kFull, d, 31);
    }
  }
  __syncthreads();
}

// Swizzled scales are limited to S <= 2^27 - 4 columns (2^25 - 1 four-column
// tiles): the gather counts the 4-byte words of a 128-row output block,
// 128 ceil(S/4), in 32 bits (2^25 tiles would make that count wrap to 0), and
// the padding writer the padded width 4 ceil(S/4).
constexpr uint32_t kMaxSwizzleTileCols = (1u << 25) - 1;

// Staging tile of the aligned path of mx_swizzle_experts_kernel: 128 rows x
// 32 words (128 scale columns), row pitch 33 words plus 8 more words per
// 32-row quarter. A warp that writes one row's 32 words, and a warp that reads
// one word from each of the 32 rows {b .. b+7} + {0, 32, 64, 96} (one swizzled
// output line), then touches 32 different banks.
constexpr uint32_t kSwzChunkWords = 32;
constexpr uint32_t kSwzPitch = kSwzChunkWords + 1;
__device__ __forceinline__ uint32_t swz_tile_index(uint32_t r, uint32_t c) {
  return r * kSwzPitch + (r >> 5) * 8 + c;
}

// Per-expert swizzled scales of a stacked tensor, gathered from its compact
// scales [M, S] (written by the quantize launch just before, in stream
// order): output block i (128 padded rows x Sp = 4 ceil(S/4) columns, at
// byte 128 i Sp) belongs to the expert e with pb[e] <= 128 i < pb[e + 1] and
// holds that expert's rows off[e] + 128 i - pb[e] .. +127; rows past the
// expert's end and columns past S are 0x00. Persistent CTAs build the row
// table once, then write whole blocks in output order. No byte at or past
// `cap` is written, whatever the offsets hold.
//  - words_aligned (S % 4 == 0, 4-byte aligned scales): a block goes through
//    shared memory in chunks of 32 words (128 columns) per row: each warp
//    reads whole row segments (coalesced), then each thread writes one output
//    word (four scale columns of one row) of the swizzled lines.
//  - otherwise each thread gathers its output words byte by byte from the
//    compact rows.
__global__ void __launch_bounds__(kThreads, 4)
mx_swizzle_experts_kernel(const uint8_t* __restrict__ scale, uint8_t* __restrict__ swz,
                          const int64_t* __restrict__ offs, int32_t E, int64_t M, uint32_t S,
                          uint32_t Sp4, uint64_t cap, bool words_aligned) {
  pdl_enter();
  extern __shared__ int64_t s_rows[];
  __shared__ uint32_t tile[128 * kSwzPitch + 3 * 8];
  int64_t* off = s_rows;
  int64_t* pb = s_rows + (E + 1);
  load_expert_rows(offs, E, M, off, pb);
  const uint64_t blocks = uint64_t(pb[E]) >> 7;
  const uint32_t words = 128 * Sp4;  // 4-byte words per output block
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto store_word = [&](uint64_t o, uint32_t v) {
    if (o + 4 <= cap) {
      st_u32(swz + o, v);
    } else {
#pragma unroll
      for (uint32_t k = 0; k < 4; k++)
        if (o + k < cap) st_u8(swz + o + k, (v >> (8 * k)) & 0xffu);
    }
  };
  for (uint64_t i = blockIdx.x; i < blocks; i += gridDim.x) {
    const int64_t prow = int64_t(i) << 7;
    int lo = 0, hi = E;  // invariant: pb[lo] <= prow < pb[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pb[mid] <= prow) lo = mid; else hi = mid;
    }
    const int64_t r0 = off[lo] + (prow - pb[lo]);  // first source row of the block
    const int64_t rend = off[lo + 1];
    if (words_aligned) {
      // rows r0 .. r0 + nrows - 1 exist (1 <= nrows <= 128: the block lies in
      // expert lo's padded rows, which start on its first row)
      const int64_t left = rend - r0;
      const uint32_t nrows = left < 128 ? uint32_t(left < 0 ? 0 : left) : 128u;
      const uint32_t* src = reinterpret_cast<const uint32_t*>(scale);  // S / 4 = Sp4 words a row
      for (uint32_t c0 = 0; c0 < Sp4; c0 += kSwzChunkWords) {
        const uint32_t cw = Sp4 - c0 < kSwzChunkWords ? Sp4 - c0 : kSwzChunkWords;
        // a warp takes rows warp, warp + 8, ..., eight loads in flight a lane
        constexpr uint32_t kWarps = kThreads / 32, kBatch = 8;
        const uint32_t* row_src = src + uint64_t(r0) * Sp4 + c0 + uint32_t(lane);
#pragma unroll
        for (uint32_t b = 0; b < 128 / (kWarps * kBatch); b++) {
          uint32_t v[kBatch];
#pragma unroll
          for (uint32_t k = 0; k < kBatch; k++) {
            const uint32_t r = uint32_t(warp) + (b * kBatch + k) * kWarps;
            v[k] = (r < nrows && uint32_t(lane) < cw) ? row_src[r * Sp4] : 0u;  // < 2^32: Sp4 <= 2^25
          }
#pragma unroll
          for (uint32_t k = 0; k < kBatch; k++)
            tile[swz_tile_index(uint32_t(warp) + (b * kBatch + k) * kWarps, uint32_t(lane))] = v[k];
        }
        __syncthreads();
        // output words of the chunk's tiles c0 .. c0 + cw - 1, in output order:
        // word wi of tile j holds row (wi % 4) 32 + wi / 4, columns 4 j .. 4 j + 3
        const uint64_t o0 = (i * words + uint64_t(c0) * 128) * 4;
        for (uint32_t w = threadIdx.x; w < cw * 128; w += kThreads) {
          const uint32_t jj = w >> 7, wi = w & 127;
          const uint32_t r = (wi & 3) * 32 + (wi >> 2);
          store_word(o0 + 4 * w, tile[swz_tile_index(r, jj)]);
        }
        __syncthreads();
      }
      continue;
    }
    constexpr int kU = 4;  // words per thread and round, all loaded before any is stored
    for (uint32_t w0 = threadIdx.x; w0 < words; w0 += kThreads * kU) {
      uint32_t v[kU];
#pragma unroll
      for (int u = 0; u < kU; u++) {
        const uint32_t w = w0 + u * kThreads;
        const uint32_t j = w >> 7, wi = w & 127;    // tile of 4 columns, word in the tile
        const int64_t row = r0 + int64_t((wi & 3) * 32 + (wi >> 2));
        v[u] = 0;
        if (w < words && row < rend) {
          const uint8_t* src = scale + uint64_t(row) * S + 4 * j;
#pragma unroll
          for (uint32_t k = 0; k < 4; k++)
            if (4 * j + k < S) v[u] |= uint32_t(src[k]) << (8 * k);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; u++) {
        const uint32_t w = w0 + u * kThreads;
        if (w < words) store_word((i * words + w) * 4, v[u]);
      }
    }
  }
}

// Zero bytes of the swizzled layout outside the real [M, S] scales.
template <int MAXE>
__device__ __forceinline__ void fill_swizzle_padding(const QuantArgs<MAXE>& a) {
  const uint64_t total = a.pad_a + a.pad_b;
  const uint32_t Sp = a.Sp4 * 4;
  const uint64_t stride = uint64_t(gridDim.x) * kThreads;
  for (uint64_t p = uint64_t(blockIdx.x) * kThreads + threadIdx.x; p < total; p += stride) {
    uint64_t r;
    uint32_t c;
    if (p < a.pad_a) {
      const uint32_t w = Sp - a.S;
      r = p / w;
      c = a.S + uint32_t(p % w);
    } else {
      const uint64_t t = p - a.pad_a;
      r = a.M + t / Sp;
      c = uint32_t(t % Sp);
    }
    st_u8(a.swz + swz_offset(r, c, a.Sp4), 0);
  }
}

template <typename InT, bool V8, bool STRIDED, int SWZ, int MAXE, int FMT>
__global__ void __launch_bounds__(kThreads)
mx_quant_kernel(const __grid_constant__ QuantArgs<MAXE> a) {
  pdl_enter();
  const uint32_t tile = blockIdx.x;
  int e = 0;
  if constexpr (MAXE > 1) {
    int lo = 0, hi = a.E;  // invariant: tbase[lo] <= tile < tbase[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.tbase[mid] <= tile) lo = mid; else hi = mid;
    }
    e = lo;
  }
  const uint64_t tg0 = uint64_t(tile - a.tbase[e]) * kGroupsPerTile;  // tile's first group
  const uint64_t left = a.gbase[e + 1] - a.gbase[e] - tg0;
  const uint32_t nt = left < kGroupsPerTile ? uint32_t(left) : uint32_t(kGroupsPerTile);
  const bool full = nt == kGroupsPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t half = lane & 1;
  const uint32_t lg0 = warp * kGroupsPerWarp + (lane >> 1);  // tile-local group of step 0

  const InT* x = static_cast<const InT*>(a.x[e]);
  constexpr uint32_t CB = kCodeBytes<FMT>;
  uint8_t* qt = a.q + (a.gbase[e] + tg0) * CB + half * (CB / 2);
  uint8_t* st = a.scale + a.gbase[e] + tg0;

  // row / column of the lane's group (strided input, swizzled scales)
  constexpr bool kRC = STRIDED || SWZ != kSwzNone;
  uint64_t r = 0;
  uint32_t c = 0;
  if constexpr (kRC) {
    const uint64_t g = tg0 + lg0;
    r = a.rows.div(g);
    c = uint32_t(g - r * a.S);
  }
  uint64_t rr[kSteps];
  uint32_t cc[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    rr[u] = r;
    cc[u] = c;
    if constexpr (kRC) {
      c += kGroupsPerStep;
      while (c >= a.S) {
        c -= a.S;
        ++r;
      }
    }
  }

  In16<InT> v[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lg = lg0 + u * kGroupsPerStep;
    const InT* p;
    if constexpr (STRIDED) {
      p = x + rr[u] * uint64_t(a.ld) + cc[u] * 32 + half * 16;
    } else {
      p = x + (tg0 + lg) * 32 + half * 16;
    }
    if (full || lg < nt) v[u].template load<V8>(p); else v[u].zero();
  }

#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lg = lg0 + u * kGroupsPerStep;
    float amax = v[u].absmax();
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, 0.0f);  // a group holding only NaNs has amax 0
    const uint32_t b = mx_scale_byte<kEmax<FMT>>(amax);
    uint4 o4;
    uint2 o2;
    if constexpr (FMT == kE4M3) o4 = to_e4m3(v[u], pow2_quant(b));
    else o2 = to_e2m1(v[u], pow2_quant(b));
    if (full || lg < nt) {
      if constexpr (FMT == kE4M3) st_v4(qt + lg * CB, o4);
      else st_v2(qt + lg * CB, o2);
      if (half == 0) {
        st_u8(st + lg, b);
        if constexpr (SWZ == kSwzTensor) st_u8(a.swz + swz_offset(rr[u], cc[u], a.Sp4), b);
      }
    }
  }
  if constexpr (SWZ == kSwzTensor) fill_swizzle_padding(a);
}

// ------------------------------------------------------- decode and store

// decode(code) * mul of a lane's 16 E4M3 codes (four words, first code in the
// low byte of cw[0]); exact in fp32 except for overflow to inf.
__device__ __forceinline__ void decode_e4m3_16(const uint32_t (&cw)[4], float mul,
                                               float (&f)[16]) {
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const float2 d = f16x2_to_f32x2(cvt_f16x2_from_e4m3x2(cw[k >> 1] >> (16 * (k & 1))));
    const float2 p = mul2(d.x, d.y, mul);
    f[2 * k] = p.x;
    f[2 * k + 1] = p.y;
  }
}

// The same for 16 E2M1 codes, two per byte, even element in the low nibble.
__device__ __forceinline__ void decode_e2m1_16(uint2 cw, float mul, float (&f)[16]) {
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xffu;
    const float2 d = f16x2_to_f32x2(cvt_f16x2_from_e2m1x2(byte));
    const float2 p = mul2(d.x, d.y, mul);
    f[2 * k] = p.x;
    f[2 * k + 1] = p.y;
  }
}

// True if any of the four words holds the E4M3 NaN code 0x7F or 0xFF.
__device__ __forceinline__ bool any_e4m3_nan(const uint32_t (&cw)[4]) {
  const uint32_t m = 0x7f7f7f7fu, o = 0x01010101u;
  return ((((cw[0] & m) + o) | ((cw[1] & m) + o) | ((cw[2] & m) + o) | ((cw[3] & m) + o)) &
          0x80808080u) != 0;
}

// Writes a lane's 16 fp32 values as OutT (bf16: round to nearest even). When
// `any_nan`, every element i with is_nan(i) is written as the canonical NaN
// (0x7FC0 / 0x7FC00000) instead.
template <typename OutT, bool V8, typename IsNan>
__device__ __forceinline__ void store16(OutT* dst, const float (&f)[16], bool any_nan,
                                        IsNan is_nan) {
  if constexpr (sizeof(OutT) == 2) {
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; k++) w[k] = cvt_bf16x2(f[2 * k], f[2 * k + 1]);
    if (any_nan) {
#pragma unroll
      for (int i = 0; i < 16; i++) {
        if (is_nan(i)) {
          const int sh = 16 * (i & 1);
          w[i >> 1] = (w[i >> 1] & ~(0xffffu << sh)) | (0x7fc0u << sh);
        }
      }
    }
    if constexpr (V8) {
      st_v8(dst, w);
    } else {
      st_v4(dst, make_uint4(w[0], w[1], w[2], w[3]));
      st_v4(dst + 8, make_uint4(w[4], w[5], w[6], w[7]));
    }
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; i++) w[i] = __float_as_uint(f[i]);
    if (any_nan) {
#pragma unroll
      for (int i = 0; i < 16; i++)
        if (is_nan(i)) w[i] = 0x7fc00000u;
    }
    if constexpr (V8) {
      st_v8(dst, *reinterpret_cast<const uint32_t(*)[8]>(&w[0]));
      st_v8(dst + 8, *reinterpret_cast<const uint32_t(*)[8]>(&w[8]));
    } else {
#pragma unroll
      for (int i = 0; i < 4; i++)
        st_v4(dst + 4 * i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
    }
  }
}

// ---------------------------------------------------------------- dequant

// A lane owns 16 codes (one 16-byte load of E4M3 codes, one 8-byte load of
// packed E2M1) and writes 16 outputs (32 bytes of bf16, 64 of fp32, with
// 256-bit stores when 32-byte aligned); two lanes a group; 16 groups per warp
// step. Tiles are taken from the last to the first: a dequantize that follows
// a quantize of the same codes then starts on the rows that quantize wrote
// last, much of which is still in L2 (measured 1-2 % off the pair's time).
constexpr int kDqSteps = 2;
constexpr int kDqGroupsPerWarp = 16 * kDqSteps;
constexpr int kDqGroupsPerTile = kDqGroupsPerWarp * (kThreads / 32);

template <typename OutT, bool V8, int FMT>
__global__ void __launch_bounds__(kThreads)
mx_dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scale,
                  OutT* __restrict__ y, uint64_t ng) {
  pdl_enter();
  constexpr uint32_t CB = kCodeBytes<FMT>;
  const uint64_t g0 = uint64_t(gridDim.x - 1 - blockIdx.x) * kDqGroupsPerTile;
  const uint64_t left = ng - g0;
  const uint32_t nt = left < kDqGroupsPerTile ? uint32_t(left) : uint32_t(kDqGroupsPerTile);
  const bool full = nt == kDqGroupsPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t half = lane & 1;
  const uint32_t lg0 = warp * kDqGroupsPerWarp + (lane >> 1);
  const uint8_t* qt = q + g0 * CB + half * (CB / 2);
  const uint8_t* st = scale + g0;
  OutT* yt = y + g0 * 32 + half * 16;

  uint32_t c[kDqSteps][4];
  uint32_t b[kDqSteps];
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lg = lg0 + u * 16;
    c[u][0] = c[u][1] = c[u][2] = c[u][3] = 0;
    b[u] = 127;
    if (full || lg < nt) {
      if constexpr (FMT == kE4M3) {
        const uint4 t = ld_nc_v4(qt + lg * CB);
        c[u][0] = t.x; c[u][1] = t.y; c[u][2] = t.z; c[u][3] = t.w;
      } else {
        const uint2 t = ld_nc_v2(qt + lg * CB);
        c[u][0] = t.x; c[u][1] = t.y;
      }
      b[u] = ld_nc_u8(st + lg);
    }
  }
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lg = lg0 + u * 16;
    if (!(full || lg < nt)) continue;
    const float mul = pow2_dequant(b[u]);
    const uint32_t (&cw)[4] = c[u];
    const uint32_t bu = b[u];
    float f[16];
    if constexpr (FMT == kE4M3) {
      decode_e4m3_16(cw, mul, f);
      store16<OutT, V8>(yt + lg * 32, f, any_e4m3_nan(cw) || bu == 255, [&](int i) {
        return ((cw[i >> 2] >> (8 * (i & 3))) & 0x7f) == 0x7f || bu == 255;
      });
    } else {
      // E2M1 has no NaN code: only the E8M0 NaN scale gives NaN outputs.
      decode_e2m1_16(make_uint2(cw[0], cw[1]), mul, f);
      store16<OutT, V8>(yt + lg * 32, f, bu == 255, [](int) { return true; });
    }
  }
}

// ----------------------------------------------------------- fake quantize

struct FakeArgs {
  const void* x;
  void* y;
  int64_t ld;       // input row stride in elements (STRIDED only)
  FastDiv rows;     // group index -> row
  uint32_t S;       // groups per row
  uint64_t groups;  // M * S
};

// y = decode(quantize(x)) * 2^(byte - 127) per group, quantize exactly as in
// mx_quant_kernel, decode exactly as in mx_dequant_kernel; the codes stay in
// registers. Work split as in mx_quant_kernel; y is contiguous [M, N].
template <typename InT, typename OutT, bool V8, bool STRIDED, int FMT>
__global__ void __launch_bounds__(kThreads)
mx_fake_quant_kernel(const __grid_constant__ FakeArgs a) {
  pdl_enter();
  const uint64_t tg0 = uint64_t(blockIdx.x) * kGroupsPerTile;
  const uint64_t left = a.groups - tg0;
  const uint32_t nt = left < kGroupsPerTile ? uint32_t(left) : uint32_t(kGroupsPerTile);
  const bool full = nt == kGroupsPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t half = lane & 1;
  const uint32_t lg0 = warp * kGroupsPerWarp + (lane >> 1);
  const InT* x = static_cast<const InT*>(a.x);
  OutT* yt = static_cast<OutT*>(a.y) + tg0 * 32 + half * 16;

  uint64_t r = 0;
  uint32_t c = 0;
  if constexpr (STRIDED) {
    const uint64_t g = tg0 + lg0;
    r = a.rows.div(g);
    c = uint32_t(g - r * a.S);
  }
  In16<InT> v[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lg = lg0 + u * kGroupsPerStep;
    const InT* p;
    if constexpr (STRIDED) {
      p = x + r * uint64_t(a.ld) + c * 32 + half * 16;
      c += kGroupsPerStep;
      while (c >= a.S) {
        c -= a.S;
        ++r;
      }
    } else {
      p = x + (tg0 + lg) * 32 + half * 16;
    }
    if (full || lg < nt) v[u].template load<V8>(p); else v[u].zero();
  }

#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lg = lg0 + u * kGroupsPerStep;
    float amax = v[u].absmax();
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, 0.0f);
    const uint32_t b = mx_scale_byte<kEmax<FMT>>(amax);
    const float dmul = pow2_dequant(b);
    float f[16];
    if constexpr (FMT == kE4M3) {
      const uint4 o = to_e4m3(v[u], pow2_quant(b));
      const uint32_t cw[4] = {o.x, o.y, o.z, o.w};
      decode_e4m3_16(cw, dmul, f);
      if (full || lg < nt) {
        store16<OutT, V8>(yt + lg * 32, f, any_e4m3_nan(cw), [&](int i) {
          return ((cw[i >> 2] >> (8 * (i & 3))) & 0x7f) == 0x7f;
        });
      }
    } else {
      decode_e2m1_16(to_e2m1(v[u], pow2_quant(b)), dmul, f);
      if (full || lg < nt) store16<OutT, V8>(yt + lg * 32, f, false, [](int) { return false; });
    }
  }
}

// ------------------------------------------------------------------ host

inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename InT, bool V8, bool STRIDED, int SWZ, int MAXE, int FMT>
mxq_status launch_quant(const QuantArgs<MAXE>& a, uint32_t grid, cudaStream_t stream) {
  return launched(launch_pdl(mx_quant_kernel<InT, V8, STRIDED, SWZ, MAXE, FMT>, grid, stream, a));
}

template <typename InT, bool V8, int FMT>
mxq_status dispatch_single(const QuantArgs<1>& a, bool strided, bool swz, uint32_t grid,
                           cudaStream_t s) {
  if (strided) {
    return swz ? launch_quant<InT, V8, true, kSwzTensor, 1, FMT>(a, grid, s)
               : launch_quant<InT, V8, true, kSwzNone, 1, FMT>(a, grid, s);
  }
  return swz ? launch_quant<InT, V8, false, kSwzTensor, 1, FMT>(a, grid, s)
             : launch_quant<InT, V8, false, kSwzNone, 1, FMT>(a, grid, s);
}

template <int FMT>
mxq_status quantize_impl(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                         uint8_t* q, uint8_t* scale, uint8_t* scale_swz, mxq_stream_t stream) {
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 32 != 0 || ld_x < N) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x || !q || !scale) return MXQ_ERR_NULL;
  const uint64_t S = uint64_t(N) / 32;
  const uint64_t groups = uint64_t(M) * S;
  const uint64_t tiles = (groups + kGroupsPerTile - 1) / kGroupsPerTile;
  if (S > 0xffffffffull || tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  if (scale_swz != nullptr && (S + 3) / 4 > kMaxSwizzleTileCols) return MXQ_ERR_SHAPE;
  const uint64_t row_bytes = uint64_t(ld_x) * elem_size(dt);
  if (!aligned16(x) || row_bytes % 16 != 0 || !aligned16(q)) return MXQ_ERR_ALIGN;

  QuantArgs<1> a{};
  a.q = q;
  a.scale = scale;
  a.swz = scale_swz;
  a.ld = ld_x;
  a.rows = FastDiv::make(uint32_t(S));
  a.S = uint32_t(S);
  a.Sp4 = uint32_t((S + 3) / 4);
  a.M = uint64_t(M);
  const uint64_t Mp = (uint64_t(M) + 127) / 128 * 128, Sp = uint64_t(a.Sp4) * 4;
  a.pad_a = uint64_t(M) * (Sp - S);
  a.pad_b = (Mp - uint64_t(M)) * Sp;
  a.E = 1;
  a.x[0] = x;
  a.gbase[0] = 0;
  a.gbase[1] = groups;
  a.tbase[0] = 0;
  a.tbase[1] = uint32_t(tiles);
  const bool strided = ld_x != N;
  const bool swz = scale_swz != nullptr;
  const bool v8 = aligned32(x) && row_bytes % 32 == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  if (dt == MXQ_BF16) {
    return v8 ? dispatch_single<uint16_t, true, FMT>(a, strided, swz, grid, s)
              : dispatch_single<uint16_t, false, FMT>(a, strided, swz, grid, s);
  }
  return v8 ? dispatch_single<float, true, FMT>(a, strided, swz, grid, s)
            : dispatch_single<float, false, FMT>(a, strided, swz, grid, s);
}

template <int FMT>
mxq_status dequantize_impl(const uint8_t* q, const uint8_t* scale, int64_t M, int64_t N, void* y,
                           int out_dt, mxq_stream_t stream) {
  if (!valid_dtype(out_dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 32 != 0) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!q || !scale || !y) return MXQ_ERR_NULL;
  if (!aligned16(q) || !aligned16(y)) return MXQ_ERR_ALIGN;
  const uint64_t groups = uint64_t(M) * (uint64_t(N) / 32);
  const uint64_t tiles = (groups + kDqGroupsPerTile - 1) / kDqGroupsPerTile;
  if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  const bool v8 = aligned32(y);
  if (out_dt == MXQ_BF16) {
    uint16_t* yp = static_cast<uint16_t*>(y);
    return launched(v8 ? launch_pdl(mx_dequant_kernel<uint16_t, true, FMT>, grid, s, q, scale, yp, groups)
                       : launch_pdl(mx_dequant_kernel<uint16_t, false, FMT>, grid, s, q, scale, yp, groups));
  }
  float* yp = static_cast<float*>(y);
  return launched(v8 ? launch_pdl(mx_dequant_kernel<float, true, FMT>, grid, s, q, scale, yp, groups)
                     : launch_pdl(mx_dequant_kernel<float, false, FMT>, grid, s, q, scale, yp, groups));
}

template <int MAXE, int FMT>
mxq_status grouped_impl(int32_t E, const void* const* xs, const int64_t* rows, int64_t N,
                        int dt, uint8_t* q, uint8_t* scale, cudaStream_t stream) {
  QuantArgs<MAXE> a{};
  const uint64_t S = uint64_t(N) / 32;
  uint64_t groups = 0, tiles = 0;
  bool v8 = true;
  a.E = E;
  for (int32_t e = 0; e < E; e++) {
    a.x[e] = xs[e];
    a.gbase[e] = groups;
    a.tbase[e] = uint32_t(tiles);
    const uint64_t ng = uint64_t(rows[e]) * S;
    if (ng && !aligned32(xs[e])) v8 = false;
    groups += ng;
    tiles += (ng + kGroupsPerTile - 1) / kGroupsPerTile;
    if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  }
  a.gbase[E] = groups;
  a.tbase[E] = uint32_t(tiles);
  if (tiles == 0) return MXQ_OK;
  a.q = q;
  a.scale = scale;
  a.S = uint32_t(S);
  const uint32_t grid = uint32_t(tiles);
  if (dt == MXQ_BF16) {
    return v8 ? launch_quant<uint16_t, true, false, kSwzNone, MAXE, FMT>(a, grid, stream)
              : launch_quant<uint16_t, false, false, kSwzNone, MAXE, FMT>(a, grid, stream);
  }
  return v8 ? launch_quant<float, true, false, kSwzNone, MAXE, FMT>(a, grid, stream)
            : launch_quant<float, false, false, kSwzNone, MAXE, FMT>(a, grid, stream);
}

template <int FMT>
mxq_status grouped_entry(int32_t E, const void* const* xs, const int64_t* rows, int64_t N,
                         int dt, uint8_t* q, uint8_t* scale, mxq_stream_t stream) {
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (E < 1 || E > MXQ_GROUPED_MAX_EXPERTS || N < 0 || N % 32 != 0) return MXQ_ERR_SHAPE;
  if (!xs || !rows) return MXQ_ERR_NULL;
  if (uint64_t(N) / 32 > 0xffffffffull) return MXQ_ERR_SHAPE;
  int64_t total = 0;
  for (int32_t e = 0; e < E; e++) {
    if (rows[e] < 0) return MXQ_ERR_SHAPE;
    if (rows[e] > 0 && N > 0) {
      if (!xs[e]) return MXQ_ERR_NULL;
      if (!aligned16(xs[e])) return MXQ_ERR_ALIGN;
    }
    total += rows[e];
  }
  if (total == 0 || N == 0) return MXQ_OK;
  if (!q || !scale) return MXQ_ERR_NULL;
  if (!aligned16(q)) return MXQ_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (E <= 64) return grouped_impl<64, FMT>(E, xs, rows, N, dt, q, scale, s);
  return grouped_impl<MXQ_GROUPED_MAX_EXPERTS, FMT>(E, xs, rows, N, dt, q, scale, s);
}

// Grouped quantize of a stacked tensor: the compact outputs are those of the
// flattened [M, N] call (groups never cross rows, so expert boundaries change
// no byte of them), in one launch; with scale_swz a second launch gathers
// each expert's scales into its own swizzled block, placed by the device row
// offsets.
template <int FMT>
mxq_status grouped_stacked_entry(const void* x, int dt, int32_t E, const int64_t* row_offsets,
                                 int64_t M, int64_t N, uint8_t* q, uint8_t* scale,
                                 uint8_t* scale_swz, int64_t swz_bytes, mxq_stream_t stream) {
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (E < 1 || E > MXQ_GROUPED_MAX_EXPERTS || M < 0 || N < 0 || N % 32 != 0) return MXQ_ERR_SHAPE;
  if (!row_offsets) return MXQ_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(row_offsets) & 7u) return MXQ_ERR_ALIGN;
  if (scale_swz && swz_bytes < 0) return MXQ_ERR_SHAPE;
  if (scale_swz && !aligned16(scale_swz)) return MXQ_ERR_ALIGN;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x || !q || !scale) return MXQ_ERR_NULL;
  const uint64_t S = uint64_t(N) / 32;
  const uint64_t groups = uint64_t(M) * S;
  const uint64_t tiles = (groups + kGroupsPerTile - 1) / kGroupsPerTile;
  if (S > 0xffffffffull || tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  if (scale_swz != nullptr && (S + 3) / 4 > kMaxSwizzleTileCols) return MXQ_ERR_SHAPE;
  const uint64_t row_bytes = uint64_t(N) * elem_size(dt);
  if (!aligned16(x) || row_bytes % 16 != 0 || !aligned16(q)) return MXQ_ERR_ALIGN;
  QuantArgs<1> a{};
  a.q = q;
  a.scale = scale;
  a.ld = N;
  a.rows = FastDiv::make(uint32_t(S));
  a.S = uint32_t(S);
  a.M = uint64_t(M);
  a.E = 1;
  a.x[0] = x;
  a.gbase[0] = 0;
  a.gbase[1] = groups;
  a.tbase[0] = 0;
  a.tbase[1] = uint32_t(tiles);
  const bool v8 = aligned32(x) && row_bytes % 32 == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  mxq_status st;
  if (dt == MXQ_BF16)
    st = v8 ? launch_quant<uint16_t, true, false, kSwzNone, 1, FMT>(a, grid, s)
            : launch_quant<uint16_t, false, false, kSwzNone, 1, FMT>(a, grid, s);
  else
    st = v8 ? launch_quant<float, true, false, kSwzNone, 1, FMT>(a, grid, s)
            : launch_quant<float, false, false, kSwzNone, 1, FMT>(a, grid, s);
  if (st != MXQ_OK || scale_swz == nullptr) return st;
  // the gather: as many persistent CTAs as there can be output blocks, up to
  // four per multiprocessor
  const uint32_t Sp4 = uint32_t((S + 3) / 4);
  const uint64_t max_blocks = (uint64_t(M) + 127 * uint64_t(E)) / 128;
  const uint64_t cap_ctas = uint64_t(sm_count()) * 4;
  const uint32_t sgrid = uint32_t(std::max<uint64_t>(1, std::min(max_blocks, cap_ctas)));
  const size_t smem = 2 * sizeof(int64_t) * size_t(E + 1);
  const bool words_aligned = S % 4 == 0 && (reinterpret_cast<uintptr_t>(scale) & 3u) == 0;
  return launched(launch_pdl_ex(mx_swizzle_experts_kernel, sgrid, kThreads, smem, s,
                                static_cast<const uint8_t*>(scale), scale_swz, row_offsets, E,
                                int64_t(M), uint32_t(S), Sp4, uint64_t(swz_bytes), words_aligned));
}

template <typename InT, typename OutT, int FMT>
mxq_status launch_fake(const FakeArgs& a, bool v8, bool strided, uint32_t grid, cudaStream_t s) {
  if (v8) {
    return launched(strided ? launch_pdl(mx_fake_quant_kernel<InT, OutT, true, true, FMT>, grid, s, a)
                            : launch_pdl(mx_fake_quant_kernel<InT, OutT, true, false, FMT>, grid, s, a));
  }
  return launched(strided ? launch_pdl(mx_fake_quant_kernel<InT, OutT, false, true, FMT>, grid, s, a)
                          : launch_pdl(mx_fake_quant_kernel<InT, OutT, false, false, FMT>, grid, s, a));
}

template <int FMT>
mxq_status fake_dispatch(const FakeArgs& a, int dt, int out_dt, bool v8, bool strided,
                         uint32_t grid, cudaStream_t s) {
  if (dt == MXQ_BF16) {
    return out_dt == MXQ_BF16 ? launch_fake<uint16_t, uint16_t, FMT>(a, v8, strided, grid, s)
                              : launch_fake<uint16_t, float, FMT>(a, v8, strided, grid, s);
  }
  return out_dt == MXQ_BF16 ? launch_fake<float, uint16_t, FMT>(a, v8, strided, grid, s)
                            : launch_fake<float, float, FMT>(a, v8, strided, grid, s);
}

}  // namespace
}  // namespace mxq

extern "C" {

mxq_status mxfp8_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* qweight, uint8_t* scale, uint8_t* scale_swz,
                          mxq_stream_t stream) {
  return mxq::quantize_impl<mxq::kE4M3>(x, dt, M, N, ld_x, qweight, scale, scale_swz, stream);
}

mxq_status mxfp8_dequantize(const uint8_t* qweight, const uint8_t* scale, int64_t M,
                            int64_t N, void* y, int out_dt, mxq_stream_t stream) {
  return mxq::dequantize_impl<mxq::kE4M3>(qweight, scale, M, N, y, out_dt, stream);
}

mxq_status mxfp8_quantize_grouped(const void* x, int dt, int32_t E, const int64_t* row_offsets,
                                  int64_t M_total, int64_t N, uint8_t* qweight, uint8_t* scale,
                                  mxq_stream_t stream) {
  return mxq::grouped_stacked_entry<mxq::kE4M3>(x, dt, E, row_offsets, M_total, N, qweight, scale,
                                                nullptr, 0, stream);
}

mxq_status mxfp8_quantize_grouped_swizzled(const void* x, int dt, int32_t E,
                                           const int64_t* row_offsets, int64_t M_total, int64_t N,
                                           uint8_t* qweight, uint8_t* scale, uint8_t* scale_swz,
                                           int64_t swz_bytes, mxq_stream_t stream) {
  if (!scale_swz) return MXQ_ERR_NULL;
  return mxq::grouped_stacked_entry<mxq::kE4M3>(x, dt, E, row_offsets, M_total, N, qweight, scale,
                                                scale_swz, swz_bytes, stream);
}

mxq_status mxq_swizzle_scales(const uint8_t* scale, int64_t M, int64_t S, uint8_t* scale_swz,
                              mxq_stream_t stream) {
  using namespace mxq;
  if (M < 0 || S < 0 || (S + 3) / 4 > kMaxSwizzleTileCols) return MXQ_ERR_SHAPE;
  if (M == 0 || S == 0) return MXQ_OK;
  if (!scale || !scale_swz) return MXQ_ERR_NULL;
  if (!aligned16(scale_swz)) return MXQ_ERR_ALIGN;
  // the one-expert case of the per-expert gather: its row table is {0, M},
  // so the offsets pointer is never read
  const uint32_t Sp4 = uint32_t((S + 3) / 4);
  const uint64_t blocks = (uint64_t(M) + 127) / 128;
  const uint32_t grid = uint32_t(std::max<uint64_t>(1, std::min(blocks, uint64_t(sm_count()) * 4)));
  const uint64_t bytes = blocks * 128 * uint64_t(Sp4) * 4;
  const bool words_aligned = S % 4 == 0 && (reinterpret_cast<uintptr_t>(scale) & 3u) == 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return launched(launch_pdl_ex(mx_swizzle_experts_kernel, grid, kThreads, 2 * sizeof(int64_t) * 2, s,
                                scale, scale_swz, static_cast<const int64_t*>(nullptr), int32_t(1),
                                M, uint32_t(S), Sp4, bytes, words_aligned));
}

mxq_status mxfp8_quantize_grouped_ptrs(int32_t E, const void* const* xs, const int64_t* rows,
                                       int64_t N, int dt, uint8_t* qweight, uint8_t* scale,
                                       mxq_stream_t stream) {
  return mxq::grouped_entry<mxq::kE4M3>(E, xs, rows, N, dt, qweight, scale, stream);
}

mxq_status mxfp4_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* packed, uint8_t* scale, uint8_t* scale_swz,
                          mxq_stream_t stream) {
  return mxq::quantize_impl<mxq::kE2M1>(x, dt, M, N, ld_x, packed, scale, scale_swz, stream);
}

mxq_status mxfp4_dequantize(const uint8_t* packed, const uint8_t* scale, int64_t M, int64_t N,
                            void* y, int out_dt, mxq_stream_t stream) {
  return mxq::dequantize_impl<mxq::kE2M1>(packed, scale, M, N, y, out_dt, stream);
}

mxq_status mxfp4_quantize_grouped(const void* x, int dt, int32_t E, const int64_t* row_offsets,
                                  int64_t M_total, int64_t N, uint8_t* packed, uint8_t* scale,
                                  mxq_stream_t stream) {
  return mxq::grouped_stacked_entry<mxq::kE2M1>(x, dt, E, row_offsets, M_total, N, packed, scale,
                                                nullptr, 0, stream);
}

mxq_status mxfp4_quantize_grouped_swizzled(const void* x, int dt, int32_t E,
                                           const int64_t* row_offsets, int64_t M_total, int64_t N,
                                           uint8_t* packed, uint8_t* scale, uint8_t* scale_swz,
                                           int64_t swz_bytes, mxq_stream_t stream) {
  if (!scale_swz) return MXQ_ERR_NULL;
  return mxq::grouped_stacked_entry<mxq::kE2M1>(x, dt, E, row_offsets, M_total, N, packed, scale,
                                                scale_swz, swz_bytes, stream);
}

mxq_status mxfp4_quantize_grouped_ptrs(int32_t E, const void* const* xs, const int64_t* rows,
                                       int64_t N, int dt, uint8_t* packed, uint8_t* scale,
                                       mxq_stream_t stream) {
  return mxq::grouped_entry<mxq::kE2M1>(E, xs, rows, N, dt, packed, scale, stream);
}

mxq_status mx_fake_quantize(int fmt, const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                            void* y, int out_dt, mxq_stream_t stream) {
  using namespace mxq;
  if (fmt != MXQ_FMT_MXFP8 && fmt != MXQ_FMT_MXFP4) return MXQ_ERR_ARG;
  if (!valid_dtype(dt) || !valid_dtype(out_dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 32 != 0 || ld_x < N) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x || !y) return MXQ_ERR_NULL;
  const uint64_t S = uint64_t(N) / 32;
  const uint64_t groups = uint64_t(M) * S;
  const uint64_t tiles = (groups + kGroupsPerTile - 1) / kGroupsPerTile;
  if (S > 0xffffffffull || tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  const uint64_t row_bytes = uint64_t(ld_x) * elem_size(dt);
  if (!aligned16(x) || row_bytes % 16 != 0 || !aligned16(y)) return MXQ_ERR_ALIGN;
  FakeArgs a{};
  a.x = x;
  a.y = y;
  a.ld = ld_x;
  a.rows = FastDiv::make(uint32_t(S));
  a.S = uint32_t(S);
  a.groups = groups;
  const bool v8 = aligned32(x) && row_bytes % 32 == 0 && aligned32(y);
  const bool strided = ld_x != N;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  return fmt == MXQ_FMT_MXFP8 ? fake_dispatch<kE4M3>(a, dt, out_dt, v8, strided, grid, s)
                              : fake_dispatch<kE2M1>(a, dt, out_dt, v8, strided, grid, s);
}

}  // extern "C"
