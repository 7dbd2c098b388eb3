// nvfp4.cu -- NVFP4 two-level quantize (tensor amax pass + block pass) and
// dequantize, for sm_100a.
//
// Method ("Add FP8, NVFP4, and QARL training and export", review "What looked
// solid": two-level global + FP8-block scaling, effective = block_scale *
// global_scale, zero blocks guarded; "V4 mxfp4 #1372", review of
// fp4_act_quant: E2M1 packed two per byte, N % block_size == 0), in fp32:
//   g     = A / 2688                       A = max |x| over non-NaN elements
//   s_b   = E4M3(amax_b / (6 g))           per block of 16, RNE, saturating
//   eff   = decode(s_b) * g
//   q_i   = E2M1(x_i / eff)                correctly rounded quotient, then RNE
//                                          (|u| > 6 -> 6, NaN -> +6), or a
//                                          sign-kept zero when eff == 0
//   packed byte k of a row = q[2k] | q[2k+1] << 4.
// Divisions use __fdiv_rn (IEEE), products __fmul_rn: the kernel performs the
// same fp32 operations in the same order as the definition, so every code is
// bit-identical to it.
//
// Passes: the tensor amax must be known before any block can be quantized,
// so a first kernel reduces |x| into per-CTA partial maxima (workspace), and
// the block kernel reduces those partials itself (a few KB per CTA, from L2)
// before its first block. The block kernel walks the tiles in reverse order,
// so its first reads hit the tail of the tensor that the amax pass left in
// the 126 MB L2.
//
// Work split of the block pass: a lane owns 8 consecutive elements, two lanes
// one block of 16, a warp 16 consecutive blocks per step (512 contiguous bytes
// of bf16 in, 128 bytes of packed codes out) and kSteps steps.
#include "common.cuh"

namespace mxq {
namespace {

constexpr int kMaxPartials = 2048;  // CTAs of the amax pass (workspace floats)
constexpr int kAmaxSteps = 4;       // 8-element chunks per thread per iteration
constexpr int kSteps = 4;
constexpr int kBlocksPerWarp = 16 * kSteps;
constexpr int kBlocksPerTile = kBlocksPerWarp * (kThreads / 32);

enum GMode { kFromPartials = 0, kGiven = 1, kFromAmax = 2 };

__device__ __forceinline__ float decode_e4m3(uint32_t code) {
  return f16x2_to_f32x2(cvt_f16x2_from_e4m3x2(code)).x;
}

// ------------------------------------------------------------- amax pass

template <typename InT, bool STRIDED>
__global__ void __launch_bounds__(kThreads)
nvfp4_amax_kernel(const InT* __restrict__ x, uint64_t nchunks, uint32_t cpr, FastDiv rowdiv,
                  int64_t ld, float* __restrict__ partials) {
  __shared__ float red[kThreads / 32];
  float m = 0.0f;
  const uint64_t per_iter = uint64_t(gridDim.x) * kThreads * kAmaxSteps;
  for (uint64_t base = uint64_t(blockIdx.x) * kThreads * kAmaxSteps; base < nchunks;
       base += per_iter) {
    In8<InT> v[kAmaxSteps];
#pragma unroll
    for (int u = 0; u < kAmaxSteps; u++) {
      const uint64_t c = base + uint64_t(u) * kThreads + threadIdx.x;
      if (c < nchunks) {
        uint64_t off;
        if constexpr (STRIDED) {
          const uint64_t r = rowdiv.div(c);
          off = r * uint64_t(ld) + (c - r * cpr) * 8;
        } else {
          off = c * 8;
        }
        v[u].load(x + off);
      } else {
        v[u].zero();
      }
    }
#pragma unroll
    for (int u = 0; u < kAmaxSteps; u++) m = fmaxf(m, v[u].absmax());
  }
  m = block_max(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// One CTA: max over the partials into *amax.
__global__ void __launch_bounds__(kThreads)
nvfp4_amax_finalize_kernel(const float* __restrict__ partials, uint32_t n, float* amax) {
  __shared__ float red[kThreads / 32];
  float m = 0.0f;
  for (uint32_t i = threadIdx.x; i < n; i += kThreads) m = fmaxf(m, partials[i]);
  m = block_max(m, red);
  if (threadIdx.x == 0) *amax = m;
}

// ------------------------------------------------------------ block pass

struct QuantArgs {
  const void* x;
  int64_t ld;               // input row stride (STRIDED)
  FastDiv rowdiv;           // block index -> row (divides by bpr)
  uint32_t bpr;             // blocks per row
  uint8_t* packed;
  uint8_t* bscale;
  float* gs;                // global scale (out, or in for kGiven)
  const float* amax_in;     // kFromAmax
  const float* partials;    // kFromPartials
  uint32_t npartials;
  uint64_t nblocks;
  uint32_t ntiles;
};

template <typename InT, bool STRIDED, int GMODE>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_kernel(const __grid_constant__ QuantArgs a) {
  __shared__ float red[kThreads / 32];
  const uint32_t tile = a.ntiles - 1 - blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 1;
  const uint64_t b0 = uint64_t(tile) * kBlocksPerTile + warp * kBlocksPerWarp + (lane >> 1);
  const InT* x = static_cast<const InT*>(a.x);

  In8<InT> v[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t blk = b0 + 16 * u;
    if (blk < a.nblocks) {
      uint64_t off;
      if constexpr (STRIDED) {
        const uint64_t r = a.rowdiv.div(blk);
        off = r * uint64_t(a.ld) + (blk - r * a.bpr) * 16;
      } else {
        off = blk * 16;
      }
      v[u].load(x + off + sub * 8);
    } else {
      v[u].zero();
    }
  }

  float g;
  if constexpr (GMODE == kGiven) {
    g = *a.gs;
  } else {
    float A;
    if constexpr (GMODE == kFromAmax) {
      A = *a.amax_in;
    } else {
      float m = 0.0f;
      for (uint32_t i = threadIdx.x; i < a.npartials; i += kThreads) m = fmaxf(m, a.partials[i]);
      A = block_max(m, red);
    }
    g = __fdiv_rn(A, 2688.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.gs = g;
  }
  const bool gzero = (g == 0.0f);
  const float t = __fmul_rn(6.0f, g);

#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t blk = b0 + 16 * u;
    float amax = v[u].absmax();
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, 0.0f);  // a block holding only NaNs has amax 0
    uint32_t sb = 0;
    float eff = 0.0f;
    if (!gzero) {
      const float s = __fdiv_rn(amax, t);
      sb = isnan(s) ? 0x7fu : (cvt_e4m3x2(s, 0.0f) & 0xffu);
      eff = __fmul_rn(decode_e4m3(sb), g);
    }
    uint32_t word = 0;
    if (eff == 0.0f) {
      // zero-block guard: codes are zeros carrying the sign of x
#pragma unroll
      for (int i = 0; i < 8; i++) word |= (__float_as_uint(v[u][i]) >> 31) << (4 * i + 3);
    } else {
#pragma unroll
      for (int k = 0; k < 4; k++) {
        // fminf maps NaN to 6 (and leaves the saturation to the cvt otherwise)
        const float q0 = fminf(__fdiv_rn(v[u][2 * k], eff), 6.0f);
        const float q1 = fminf(__fdiv_rn(v[u][2 * k + 1], eff), 6.0f);
        word |= cvt_e2m1x2(q0, q1) << (8 * k);
      }
    }
    if (blk < a.nblocks) {
      st_u32(a.packed + blk * 8 + sub * 4, word);
      if (sub == 0) st_u8(a.bscale + blk, sb);
    }
  }
}

// --------------------------------------------------------------- dequant

template <typename OutT>
__global__ void __launch_bounds__(kThreads)
nvfp4_dequant_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ bscale,
                     const float* __restrict__ gs, OutT* __restrict__ y, uint64_t nblocks) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, sub = lane & 1;
  const uint64_t b0 =
      uint64_t(blockIdx.x) * kBlocksPerTile + warp * kBlocksPerWarp + (lane >> 1);
  uint32_t w[kSteps], sb[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t blk = b0 + 16 * u;
    if (blk < nblocks) {
      w[u] = ld_nc_u32(packed + blk * 8 + sub * 4);
      sb[u] = ld_nc_u8(bscale + blk);
    } else {
      w[u] = 0;
      sb[u] = 0;
    }
  }
  const float g = *gs;
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint64_t blk = b0 + 16 * u;
    if (blk >= nblocks) continue;
    const float eff = __fmul_rn(decode_e4m3(sb[u]), g);
    float f[8];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float2 p = f16x2_to_f32x2(cvt_f16x2_from_e2m1x2((w[u] >> (8 * k)) & 0xffu));
      f[2 * k] = __fmul_rn(p.x, eff);
      f[2 * k + 1] = __fmul_rn(p.y, eff);
    }
    if (!isfinite(eff)) {  // only then can a product be NaN (0 * inf, NaN scale)
#pragma unroll
      for (int i = 0; i < 8; i++)
        if (isnan(f[i])) f[i] = __uint_as_float(0x7fc00000u);
    }
    OutT* dst = y + blk * 16 + sub * 8;
    if constexpr (sizeof(OutT) == 2) {
      uint4 o = make_uint4(cvt_bf16x2(f[0], f[1]), cvt_bf16x2(f[2], f[3]),
                           cvt_bf16x2(f[4], f[5]), cvt_bf16x2(f[6], f[7]));
      if (!isfinite(eff)) {
        uint32_t ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
          if (isnan(f[i])) {
            const int sh = 16 * (i & 1);
            ow[i >> 1] = (ow[i >> 1] & ~(0xffffu << sh)) | (0x7fc0u << sh);
          }
        }
        o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
      st_v4(dst, o);
    } else {
      st_v4(dst, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                            __float_as_uint(f[2]), __float_as_uint(f[3])));
      st_v4(dst + 4, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]),
                                __float_as_uint(f[6]), __float_as_uint(f[7])));
    }
  }
}

// ------------------------------------------------------------------ host

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Launches the amax pass into `partials`; returns the number of partials.
mxq_status launch_amax(const void* x, int dt, int64_t M, int64_t N, int64_t ld, float* partials,
                       uint32_t* npartials, cudaStream_t s) {
  const uint64_t cpr = uint64_t(N) / 8;
  const uint64_t nchunks = uint64_t(M) * cpr;
  const uint64_t per_cta = uint64_t(kThreads) * kAmaxSteps;
  uint64_t grid = (nchunks + per_cta - 1) / per_cta;
  const uint64_t cap = std::min<uint64_t>(kMaxPartials, uint64_t(sm_count()) * 8);
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const FastDiv rd = FastDiv::make(uint32_t(cpr));
  const bool strided = ld != N;
  if (dt == MXQ_BF16) {
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    if (strided) nvfp4_amax_kernel<uint16_t, true><<<uint32_t(grid), kThreads, 0, s>>>(xp, nchunks, uint32_t(cpr), rd, ld, partials);
    else nvfp4_amax_kernel<uint16_t, false><<<uint32_t(grid), kThreads, 0, s>>>(xp, nchunks, uint32_t(cpr), rd, ld, partials);
  } else {
    const float* xp = static_cast<const float*>(x);
    if (strided) nvfp4_amax_kernel<float, true><<<uint32_t(grid), kThreads, 0, s>>>(xp, nchunks, uint32_t(cpr), rd, ld, partials);
    else nvfp4_amax_kernel<float, false><<<uint32_t(grid), kThreads, 0, s>>>(xp, nchunks, uint32_t(cpr), rd, ld, partials);
  }
  *npartials = uint32_t(grid);
  return check_launch();
}

template <typename InT, bool STRIDED>
mxq_status launch_quant_mode(const QuantArgs& a, int mode, cudaStream_t s) {
  switch (mode) {
    case kGiven: nvfp4_quant_kernel<InT, STRIDED, kGiven><<<a.ntiles, kThreads, 0, s>>>(a); break;
    case kFromAmax: nvfp4_quant_kernel<InT, STRIDED, kFromAmax><<<a.ntiles, kThreads, 0, s>>>(a); break;
    default: nvfp4_quant_kernel<InT, STRIDED, kFromPartials><<<a.ntiles, kThreads, 0, s>>>(a); break;
  }
  return check_launch();
}

mxq_status check_input(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x) {
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 16 != 0 || ld_x < N) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x) return MXQ_ERR_NULL;
  const uint64_t nblocks = uint64_t(M) * (uint64_t(N) / 16);
  if (uint64_t(N) / 8 > 0xffffffffull || (nblocks + kBlocksPerTile - 1) / kBlocksPerTile > 0x7fffffffull)
    return MXQ_ERR_SHAPE;
  if (!aligned16(x) || (uint64_t(ld_x) * elem_size(dt)) % 16 != 0) return MXQ_ERR_ALIGN;
  return MXQ_OK;
}

}  // namespace
}  // namespace mxq

extern "C" {

size_t mxq_nvfp4_workspace_bytes(int64_t M, int64_t N) {
  (void)M;
  (void)N;
  return sizeof(float) * mxq::kMaxPartials;
}

mxq_status nvfp4_amax(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x, float* amax,
                      void* workspace, size_t ws_bytes, mxq_stream_t stream) {
  using namespace mxq;
  mxq_status st = check_input(x, dt, M, N, ld_x);
  if (st != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!amax) return MXQ_ERR_NULL;
  if (!workspace || ws_bytes < mxq_nvfp4_workspace_bytes(M, N) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3u))
    return MXQ_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t np = 0;
  st = launch_amax(x, dt, M, N, ld_x, static_cast<float*>(workspace), &np, s);
  if (st != MXQ_OK) return st;
  nvfp4_amax_finalize_kernel<<<1, kThreads, 0, s>>>(static_cast<float*>(workspace), np, amax);
  return check_launch();
}

mxq_status nvfp4_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* packed, uint8_t* block_scale, float* global_scale,
                          const float* amax_in, uint32_t flags, void* workspace,
                          size_t ws_bytes, mxq_stream_t stream) {
  using namespace mxq;
  if (flags & ~MXQ_NVFP4_GLOBAL_GIVEN) return MXQ_ERR_ARG;
  const bool given = (flags & MXQ_NVFP4_GLOBAL_GIVEN) != 0;
  if (given && amax_in) return MXQ_ERR_ARG;
  mxq_status st = check_input(x, dt, M, N, ld_x);
  if (st != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!packed || !block_scale || !global_scale) return MXQ_ERR_NULL;
  if (!aligned16(packed)) return MXQ_ERR_ALIGN;
  const bool pass1 = !given && !amax_in;
  if (pass1 && (!workspace || ws_bytes < mxq_nvfp4_workspace_bytes(M, N) ||
                (reinterpret_cast<uintptr_t>(workspace) & 3u)))
    return MXQ_ERR_WORKSPACE;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QuantArgs a{};
  a.x = x;
  a.ld = ld_x;
  a.bpr = uint32_t(uint64_t(N) / 16);
  a.rowdiv = FastDiv::make(a.bpr);
  a.packed = packed;
  a.bscale = block_scale;
  a.gs = global_scale;
  a.amax_in = amax_in;
  a.nblocks = uint64_t(M) * a.bpr;
  a.ntiles = uint32_t((a.nblocks + kBlocksPerTile - 1) / kBlocksPerTile);
  int mode = given ? kGiven : (amax_in ? kFromAmax : kFromPartials);
  if (pass1) {
    a.partials = static_cast<const float*>(workspace);
    st = launch_amax(x, dt, M, N, ld_x, static_cast<float*>(workspace), &a.npartials, s);
    if (st != MXQ_OK) return st;
  }
  const bool strided = ld_x != N;
  if (dt == MXQ_BF16)
    return strided ? launch_quant_mode<uint16_t, true>(a, mode, s)
                   : launch_quant_mode<uint16_t, false>(a, mode, s);
  return strided ? launch_quant_mode<float, true>(a, mode, s)
                 : launch_quant_mode<float, false>(a, mode, s);
}

mxq_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* block_scale,
                            const float* global_scale, int64_t M, int64_t N, void* y,
                            int out_dt, mxq_stream_t stream) {
  using namespace mxq;
  if (!valid_dtype(out_dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 16 != 0) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!packed || !block_scale || !global_scale || !y) return MXQ_ERR_NULL;
  if (!aligned16(packed) || !aligned16(y)) return MXQ_ERR_ALIGN;
  const uint64_t nblocks = uint64_t(M) * (uint64_t(N) / 16);
  const uint64_t tiles = (nblocks + kBlocksPerTile - 1) / kBlocksPerTile;
  if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (out_dt == MXQ_BF16) {
    nvfp4_dequant_kernel<uint16_t><<<uint32_t(tiles), kThreads, 0, s>>>(
        packed, block_scale, global_scale, static_cast<uint16_t*>(y), nblocks);
  } else {
    nvfp4_dequant_kernel<float><<<uint32_t(tiles), kThreads, 0, s>>>(
        packed, block_scale, global_scale, static_cast<float*>(y), nblocks);
  }
  return check_launch();
}

}  // extern "C"
