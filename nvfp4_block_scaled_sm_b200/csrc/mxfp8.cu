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
// The hardware conversion cvt.rn.satfinite.e4m3x2.f32 rounds to nearest even
// and saturates finite and infinite values to +-448; its NaN results are
// rewritten to the canonical 0x7F.
//
// Memory layout and work split (HBM-bound: 2 bytes read, 1 + 1/32 written per
// bf16 element): a lane owns 8 consecutive elements (one 16-byte load of
// bf16, two of fp32), 4 lanes one group, a warp 8 consecutive groups per step
// (512 contiguous bytes of bf16) and kSteps steps; a CTA owns kGroupsPerTile
// consecutive groups. All kSteps loads of a lane are issued before any of
// them is used. Rows are never padded: groups do not cross rows, so the
// result for M rows equals the pad-to-32-rows-then-crop contract.
#include "common.cuh"

namespace mxq {
namespace {

constexpr int kSteps = 4;
constexpr int kGroupsPerWarp = 8 * kSteps;
constexpr int kGroupsPerTile = kGroupsPerWarp * (kThreads / 32);

// Biased E8M0 exponent of a group's amax (amax >= 0, not NaN).
__device__ __forceinline__ uint32_t e8m0_byte(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const uint32_t E = bits >> 23;
  uint32_t b = E > 8 ? E - 8 : 0;
  b = (E == 255) ? 254 : b;
  b = (bits == 0) ? 127 : b;
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

// E4M3 codes of the lane's 8 elements times `mul` (low byte = first element).
template <typename InT>
__device__ __forceinline__ uint2 to_e4m3(const In8<InT>& v, float mul) {
  uint2 o;
  o.x = cvt_e4m3x2(v[0] * mul, v[1] * mul) | (cvt_e4m3x2(v[2] * mul, v[3] * mul) << 16);
  o.y = cvt_e4m3x2(v[4] * mul, v[5] * mul) | (cvt_e4m3x2(v[6] * mul, v[7] * mul) << 16);
  return o;
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

template <typename InT, bool STRIDED, bool SWZ, int MAXE>
__global__ void __launch_bounds__(kThreads)
mxfp8_quant_kernel(const __grid_constant__ QuantArgs<MAXE> a) {
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
  const uint64_t gbeg = a.gbase[e];
  const uint64_t ng = a.gbase[e + 1] - gbeg;
  const InT* x = static_cast<const InT*>(a.x[e]);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 3;
  const uint64_t g0 =
      uint64_t(tile - a.tbase[e]) * kGroupsPerTile + warp * kGroupsPerWarp + (lane >> 2);

  In8<InT> v[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t g = g0 + 8 * u;
    if (g < ng) {
      uint64_t off;
      if constexpr (STRIDED) {
        const uint64_t r = a.rows.div(g);
        off = r * uint64_t(a.ld) + (g - r * a.S) * 32;
      } else {
        off = g * 32;
      }
      v[u].load(x + off + sub * 8);
    } else {
      v[u].zero();
    }
  }

#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t g = g0 + 8 * u;
    float amax = v[u].absmax();
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    amax = fmaxf(amax, 0.0f);  // a group holding only NaNs has amax 0
    const uint32_t b = e8m0_byte(amax);
    uint2 o = to_e4m3(v[u], pow2_quant(b));
    o.x &= ~e4m3_nan_bytes(o.x);  // NaN -> canonical 0x7F
    o.y &= ~e4m3_nan_bytes(o.y);
    if (g < ng) {
      const uint64_t go = gbeg + g;
      st_v2(a.q + go * 32 + sub * 8, o);
      if (sub == 0) {
        st_u8(a.scale + go, b);
        if constexpr (SWZ) {
          const uint64_t r = a.rows.div(g);
          st_u8(a.swz + swz_offset(r, uint32_t(g - r * a.S), a.Sp4), b);
        }
      }
    }
  }
  if constexpr (SWZ) fill_swizzle_padding(a);
}

// ---------------------------------------------------------------- dequant

// A lane owns 8 codes (one 8-byte load) and writes 8 outputs (16 bytes of
// bf16, 32 of fp32); 4 lanes one group; 8 groups per warp step.
constexpr int kDqSteps = 4;
constexpr int kDqGroupsPerWarp = 8 * kDqSteps;
constexpr int kDqGroupsPerTile = kDqGroupsPerWarp * (kThreads / 32);

template <typename OutT>
__global__ void __launch_bounds__(kThreads)
mxfp8_dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scale,
                     OutT* __restrict__ y, uint64_t ng) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 3;
  const uint64_t g0 =
      uint64_t(blockIdx.x) * kDqGroupsPerTile + warp * kDqGroupsPerWarp + (lane >> 2);
  uint2 c[kDqSteps];
  uint32_t b[kDqSteps];
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint64_t g = g0 + 8 * u;
    if (g < ng) {
      c[u] = ld_nc_v2(q + g * 32 + sub * 8);
      b[u] = ld_nc_u8(scale + g);
    } else {
      c[u] = make_uint2(0, 0);
      b[u] = 127;
    }
  }
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint64_t g = g0 + 8 * u;
    if (g >= ng) continue;
    const float mul = pow2_dequant(b[u]);
    float f[8];
    const uint32_t h[4] = {cvt_f16x2_from_e4m3x2(c[u].x), cvt_f16x2_from_e4m3x2(c[u].x >> 16),
                           cvt_f16x2_from_e4m3x2(c[u].y), cvt_f16x2_from_e4m3x2(c[u].y >> 16)};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float2 p = f16x2_to_f32x2(h[k]);
      f[2 * k] = p.x * mul;
      f[2 * k + 1] = p.y * mul;
    }
    const bool any_nan = (e4m3_nan_bytes(c[u].x) | e4m3_nan_bytes(c[u].y)) != 0 || b[u] == 255;
    OutT* dst = y + g * 32 + sub * 8;
    if constexpr (sizeof(OutT) == 2) {
      uint4 o = make_uint4(cvt_bf16x2(f[0], f[1]), cvt_bf16x2(f[2], f[3]),
                           cvt_bf16x2(f[4], f[5]), cvt_bf16x2(f[6], f[7]));
      if (any_nan) {
        uint32_t w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const uint32_t code = ((i < 4 ? c[u].x : c[u].y) >> (8 * (i & 3))) & 0x7f;
          if (code == 0x7f || b[u] == 255) {
            const int sh = 16 * (i & 1);
            w[i >> 1] = (w[i >> 1] & ~(0xffffu << sh)) | (0x7fc0u << sh);
          }
        }
        o = make_uint4(w[0], w[1], w[2], w[3]);
      }
      st_v4(dst, o);
    } else {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; i++) w[i] = __float_as_uint(f[i]);
      if (any_nan) {
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const uint32_t code = ((i < 4 ? c[u].x : c[u].y) >> (8 * (i & 3))) & 0x7f;
          if (code == 0x7f || b[u] == 255) w[i] = 0x7fc00000u;
        }
      }
      st_v4(dst, make_uint4(w[0], w[1], w[2], w[3]));
      st_v4(dst + 4, make_uint4(w[4], w[5], w[6], w[7]));
    }
  }
}

// ------------------------------------------------------------------ host

template <typename InT, bool STRIDED, bool SWZ, int MAXE>
mxq_status launch_quant(const QuantArgs<MAXE>& a, uint32_t grid, cudaStream_t stream) {
  mxfp8_quant_kernel<InT, STRIDED, SWZ, MAXE><<<grid, kThreads, 0, stream>>>(a);
  return check_launch();
}

template <typename InT>
mxq_status dispatch_single(const QuantArgs<1>& a, bool strided, bool swz, uint32_t grid,
                           cudaStream_t s) {
  if (strided) {
    return swz ? launch_quant<InT, true, true, 1>(a, grid, s)
               : launch_quant<InT, true, false, 1>(a, grid, s);
  }
  return swz ? launch_quant<InT, false, true, 1>(a, grid, s)
             : launch_quant<InT, false, false, 1>(a, grid, s);
}

template <int MAXE>
mxq_status grouped_impl(int32_t E, const void* const* xs, const int64_t* rows, int64_t N,
                        int dt, uint8_t* q, uint8_t* scale, cudaStream_t stream) {
  QuantArgs<MAXE> a{};
  const uint64_t S = uint64_t(N) / 32;
  uint64_t groups = 0, tiles = 0;
  a.E = E;
  for (int32_t e = 0; e < E; e++) {
    a.x[e] = xs[e];
    a.gbase[e] = groups;
    a.tbase[e] = uint32_t(tiles);
    const uint64_t ng = uint64_t(rows[e]) * S;
    groups += ng;
    tiles += (ng + kGroupsPerTile - 1) / kGroupsPerTile;
    if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  }
  a.gbase[E] = groups;
  a.tbase[E] = uint32_t(tiles);
  if (tiles == 0) return MXQ_OK;
  a.q = q;
  a.scale = scale;
  a.swz = nullptr;
  a.S = uint32_t(S);
  if (dt == MXQ_BF16) return launch_quant<uint16_t, false, false, MAXE>(a, uint32_t(tiles), stream);
  return launch_quant<float, false, false, MAXE>(a, uint32_t(tiles), stream);
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
  if (!aligned16(x) || (uint64_t(ld_x) * elem_size(dt)) % 16 != 0 || !aligned16(qweight))
    return MXQ_ERR_ALIGN;

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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dt == MXQ_BF16) return dispatch_single<uint16_t>(a, strided, swz, uint32_t(tiles), s);
  return dispatch_single<float>(a, strided, swz, uint32_t(tiles), s);
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
  if (out_dt == MXQ_BF16) {
    mxfp8_dequant_kernel<uint16_t><<<uint32_t(tiles), kThreads, 0, s>>>(
        qweight, scale, static_cast<uint16_t*>(y), groups);
  } else {
    mxfp8_dequant_kernel<float><<<uint32_t(tiles), kThreads, 0, s>>>(
        qweight, scale, static_cast<float*>(y), groups);
  }
  return check_launch();
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
