// mxfp8.cu -- MXFP8 rowwise quantize (compact + optional swizzled scales,
// single tensor or a group of expert tensors in one launch) and dequantize,
// for sm_100a.
//
// Method ("PR #1935 完整报告 -- Use TransformerEngine for MXFP8 quantization",
// 实现拆解 items 1 and 4; "V4 mxfp4 #1372", description): groups of 32
// consecutive elements along the last dim; per group amax = max |x| over its
// non-NaN elements, E8M0 byte = 127 for amax == 0, 254 for amax == inf, else
// clamp(E(amax) - 8, 0, 254) where E is the biased fp32 exponent field (the
// same number as floor(log2 amax) + 127 - 8, clamped; 8 = emax of E4M3), and
// q = E4M3(x * 2^(127 - byte)), round to nearest even with saturation to 448.
//
// Exactness of the fp32 path: for finite amax the byte is at most 246, so the
// multiplier 2^(127 - byte) is a normal fp32 power of two and x * multiplier
// is exact whenever the product is an fp32 normal. Products below 2^-126
// (where fp32 would round) are far below half the smallest E4M3 subnormal
// (2^-10), so they encode to a zero of the right sign either way. An infinite
// amax gives byte 254 and the subnormal multiplier 2^-127 (built from its bit
// pattern), again exact for every product that can encode to non-zero.
// cvt.rn.satfinite.e4m3x2.f32 rounds to nearest even, saturates finite and
// infinite values to +-448, keeps the sign of zero and writes every NaN as
// 0x7F (checked exhaustively against the oracle by the GPU tests).
//
// Work split (HBM-bound: 2 bytes read and 1 + 1/32 written per bf16 element):
// a lane owns 16 consecutive elements (one 256-bit load of bf16, two of fp32,
// when 32-byte aligned), two lanes a group, a warp 16 consecutive groups per
// step (1 KiB of contiguous bf16) and kSteps steps, a CTA kGroupsPerTile
// consecutive groups. All loads of a lane are issued before any is used. The
// tile's base pointers are formed once in 64-bit arithmetic; lane offsets
// inside a tile are 32-bit, and full tiles skip the bounds checks. Rows are
// never padded: groups do not cross rows, so the result for M rows equals the
// pad-to-32-rows-then-crop contract.
#include "common.cuh"

namespace mxq {
namespace {

constexpr int kGroupsPerStep = 16;  // per warp and step
constexpr int kSteps = 2;
constexpr int kGroupsPerWarp = kGroupsPerStep * kSteps;
constexpr int kGroupsPerTile = kGroupsPerWarp * (kThreads / 32);

// Biased E8M0 exponent of a group's amax (amax >= 0, not NaN).
__device__ __forceinline__ uint32_t e8m0_byte(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const uint32_t E = bits >> 23;
  uint32_t b = max(E, 8u) - 8u;
  b = (E == 255) ? 254u : b;
  b = (bits == 0) ? 127u : b;
  return b;
}

// 2^(127 - b) for b in [0, 254]; b == 254 is the fp32 subnormal 2^-127.
__device__ __forceinline__ float pow2_quant(uint32_t b) {
  return __uint_as_float(b == 254 ? 0x00400000u : (254u - b) << 23);
}

// 2^(b - 127) for a scale byte b; 0 is the fp32 subnormal 2^-127 and 255
// (the E8M0 NaN) is NaN.
__device__ __forceinline__ float pow2_dequant(uint32_t b) {
  return __uint_as_float(b == 0 ? 0x00400000u : (b == 255 ? 0x7fc00000u : b << 23));
}

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
    const float2 p = mul2(v.lo(k), v.hi(k), mul);
    c[k] = cvt_e4m3x2(p.x, p.y);
  }
  return make_uint4(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410),
                    __byte_perm(c[4], c[5], 0x5410), __byte_perm(c[6], c[7], 0x5410));
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

template <typename InT, bool V8, bool STRIDED, bool SWZ, int MAXE>
__global__ void __launch_bounds__(kThreads)
mxfp8_quant_kernel(const __grid_constant__ QuantArgs<MAXE> a) {
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
  uint8_t* qt = a.q + (a.gbase[e] + tg0) * 32 + half * 16;
  uint8_t* st = a.scale + a.gbase[e] + tg0;

  // row / column of the lane's group (strided input, swizzled scales)
  uint64_t r = 0;
  uint32_t c = 0;
  if constexpr (STRIDED || SWZ) {
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
    if constexpr (STRIDED || SWZ) {
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
    const uint32_t b = e8m0_byte(amax);
    const uint4 o = to_e4m3(v[u], pow2_quant(b));
    if (full || lg < nt) {
      st_v4(qt + lg * 32, o);
      if (half == 0) {
        st_u8(st + lg, b);
        if constexpr (SWZ) st_u8(a.swz + swz_offset(rr[u], cc[u], a.Sp4), b);
      }
    }
  }
  if constexpr (SWZ) fill_swizzle_padding(a);
}

// ---------------------------------------------------------------- dequant

// A lane owns 16 codes (one 16-byte load) and writes 16 outputs (32 bytes of
// bf16, 64 of fp32, with 256-bit stores when 32-byte aligned); two lanes a
// group; 16 groups per warp step.
constexpr int kDqSteps = 2;
constexpr int kDqGroupsPerWarp = 16 * kDqSteps;
constexpr int kDqGroupsPerTile = kDqGroupsPerWarp * (kThreads / 32);

template <typename OutT, bool V8>
__global__ void __launch_bounds__(kThreads)
mxfp8_dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scale,
                     OutT* __restrict__ y, uint64_t ng) {
  pdl_enter();
  const uint64_t g0 = uint64_t(blockIdx.x) * kDqGroupsPerTile;
  const uint64_t left = ng - g0;
  const uint32_t nt = left < kDqGroupsPerTile ? uint32_t(left) : uint32_t(kDqGroupsPerTile);
  const bool full = nt == kDqGroupsPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t half = lane & 1;
  const uint32_t lg0 = warp * kDqGroupsPerWarp + (lane >> 1);
  const uint8_t* qt = q + g0 * 32 + half * 16;
  const uint8_t* st = scale + g0;
  OutT* yt = y + g0 * 32 + half * 16;

  uint4 c[kDqSteps];
  uint32_t b[kDqSteps];
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lg = lg0 + u * 16;
    if (full || lg < nt) {
      c[u] = ld_nc_v4(qt + lg * 32);
      b[u] = ld_nc_u8(st + lg);
    } else {
      c[u] = make_uint4(0, 0, 0, 0);
      b[u] = 127;
    }
  }
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lg = lg0 + u * 16;
    if (!(full || lg < nt)) continue;
    const float mul = pow2_dequant(b[u]);
    const uint32_t cw[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
    float f[16];
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const float2 d = f16x2_to_f32x2(cvt_f16x2_from_e4m3x2(cw[k >> 1] >> (16 * (k & 1))));
      const float2 p = mul2(d.x, d.y, mul);
      f[2 * k] = p.x;
      f[2 * k + 1] = p.y;
    }
    const uint32_t m = 0x7f7f7f7fu, o = 0x01010101u;
    const bool any_nan = ((((cw[0] & m) + o) | ((cw[1] & m) + o) | ((cw[2] & m) + o) |
                           ((cw[3] & m) + o)) & 0x80808080u) != 0 || b[u] == 255;
    OutT* dst = yt + lg * 32;
    if constexpr (sizeof(OutT) == 2) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; k++) w[k] = cvt_bf16x2(f[2 * k], f[2 * k + 1]);
      if (any_nan) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
          if (((cw[i >> 2] >> (8 * (i & 3))) & 0x7f) == 0x7f || b[u] == 255) {
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
          if (((cw[i >> 2] >> (8 * (i & 3))) & 0x7f) == 0x7f || b[u] == 255) w[i] = 0x7fc00000u;
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
}

// ------------------------------------------------------------------ host

inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename InT, bool V8, bool STRIDED, bool SWZ, int MAXE>
mxq_status launch_quant(const QuantArgs<MAXE>& a, uint32_t grid, cudaStream_t stream) {
  return launched(launch_pdl(mxfp8_quant_kernel<InT, V8, STRIDED, SWZ, MAXE>, grid, stream, a));
}

template <typename InT, bool V8>
mxq_status dispatch_single(const QuantArgs<1>& a, bool strided, bool swz, uint32_t grid,
                           cudaStream_t s) {
  if (strided) {
    return swz ? launch_quant<InT, V8, true, true, 1>(a, grid, s)
               : launch_quant<InT, V8, true, false, 1>(a, grid, s);
  }
  return swz ? launch_quant<InT, V8, false, true, 1>(a, grid, s)
             : launch_quant<InT, V8, false, false, 1>(a, grid, s);
}

template <int MAXE>
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
    return v8 ? launch_quant<uint16_t, true, false, false, MAXE>(a, grid, stream)
              : launch_quant<uint16_t, false, false, false, MAXE>(a, grid, stream);
  }
  return v8 ? launch_quant<float, true, false, false, MAXE>(a, grid, stream)
            : launch_quant<float, false, false, false, MAXE>(a, grid, stream);
}

}  // namespace
}  // namespace mxq

extern "C" {

mxq_status mxfp8_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* qweight, uint8_t* scale, uint8_t* scale_swz,
                          mxq_stream_t stream) {
  using namespace mxq;
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 32 != 0 || ld_x < N) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x || !qweight || !scale) return MXQ_ERR_NULL;
  const uint64_t S = uint64_t(N) / 32;
  const uint64_t groups = uint64_t(M) * S;
  const uint64_t tiles = (groups + kGroupsPerTile - 1) / kGroupsPerTile;
  if (S > 0xffffffffull || tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  const uint64_t row_bytes = uint64_t(ld_x) * elem_size(dt);
  if (!aligned16(x) || row_bytes % 16 != 0 || !aligned16(qweight)) return MXQ_ERR_ALIGN;

  QuantArgs<1> a{};
  a.q = qweight;
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
    return v8 ? dispatch_single<uint16_t, true>(a, strided, swz, grid, s)
              : dispatch_single<uint16_t, false>(a, strided, swz, grid, s);
  }
  return v8 ? dispatch_single<float, true>(a, strided, swz, grid, s)
            : dispatch_single<float, false>(a, strided, swz, grid, s);
}

mxq_status mxfp8_dequantize(const uint8_t* qweight, const uint8_t* scale, int64_t M,
                            int64_t N, void* y, int out_dt, mxq_stream_t stream) {
  using namespace mxq;
  if (!valid_dtype(out_dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 32 != 0) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!qweight || !scale || !y) return MXQ_ERR_NULL;
  if (!aligned16(qweight) || !aligned16(y)) return MXQ_ERR_ALIGN;
  const uint64_t groups = uint64_t(M) * (uint64_t(N) / 32);
  const uint64_t tiles = (groups + kDqGroupsPerTile - 1) / kDqGroupsPerTile;
  if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  const bool v8 = aligned32(y);
  if (out_dt == MXQ_BF16) {
    uint16_t* yp = static_cast<uint16_t*>(y);
    return launched(v8 ? launch_pdl(mxfp8_dequant_kernel<uint16_t, true>, grid, s, qweight, scale, yp, groups)
                       : launch_pdl(mxfp8_dequant_kernel<uint16_t, false>, grid, s, qweight, scale, yp, groups));
  }
  float* yp = static_cast<float*>(y);
  return launched(v8 ? launch_pdl(mxfp8_dequant_kernel<float, true>, grid, s, qweight, scale, yp, groups)
                     : launch_pdl(mxfp8_dequant_kernel<float, false>, grid, s, qweight, scale, yp, groups));
}

mxq_status mxfp8_quantize_grouped(int32_t E, const void* const* xs, const int64_t* rows,
                                  int64_t N, int dt, uint8_t* qweight, uint8_t* scale,
                                  mxq_stream_t stream) {
  using namespace mxq;
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
  if (!qweight || !scale) return MXQ_ERR_NULL;
  if (!aligned16(qweight)) return MXQ_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (E <= 64) return grouped_impl<64>(E, xs, rows, N, dt, qweight, scale, s);
  return grouped_impl<MXQ_GROUPED_MAX_EXPERTS>(E, xs, rows, N, dt, qweight, scale, s);
}

}  // extern "C"
