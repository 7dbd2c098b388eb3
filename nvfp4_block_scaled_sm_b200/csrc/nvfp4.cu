// nvfp4.cu -- NVFP4 two-level quantize (tensor amax pass + block pass) and
// dequantize, for sm_100a.
//
// Method ("Add FP8, NVFP4, and QARL training and export", review "What looked
// solid": two-level global + FP8-block scaling, the effective scale being the
// block scale times the global scale, zero blocks guarded; "V4 mxfp4 #1372", review of
// fp4_act_quant: E2M1 packed two per byte, N % block_size == 0), in fp32:
//   g     = A / 2688                       A = max |x| over non-NaN elements
//   s_b   = E4M3(amax_b / (6 g))           per block of 16, RNE, saturating
//   eff   = decode(s_b) * g
//   q_i   = E2M1(x_i / eff)                correctly rounded quotient, then RNE
//                                          (|u| > 6 -> 6, NaN -> +6), or a
//                                          sign-kept zero when eff == 0
//   packed byte k of a row = q[2k] | q[2k+1] << 4.
// g, s and eff use IEEE division / multiplication (__fdiv_rn, __fmul_rn).
//
// Codes without a division per element. An E4M3 or E2M1 code is a monotone
// step function of the correctly rounded quotient f; its steps sit at the
// midpoints between neighbouring code values.
//  - E2M1 (per element): with r = rcp.approx.f32(eff) (documented error
//    <= 1 ulp), the products lo = fl(x * fl(r (1 - 2^-20))) and
//    hi = fl(x * fl(r (1 + 2^-20))) bracket f strictly (a few 2^-24 relative
//    roundings against the 2^-20 margin; f lies within 2^-24 of x / eff). When
//    E2M1(lo) == E2M1(hi) for all 16 elements, that is E2M1(f); a tie of f on
//    a midpoint puts lo and hi on opposite sides of it.
//  - E4M3 (per block): the product amax * rcp.approx(t) lies within a few
//    ulps of f; every E4M3 midpoint has at most four significant bits, so the
//    product rounds like f unless it is within 32 ulps of a value whose
//    mantissa is zero below bit 19.
// A block where either test fails (bf16 inputs make exact quotients such as
// 3.5 common), or whose divisors lie outside [2^-125, 2^125) (where the
// approximate reciprocal would not be normal), is put on a shared list and
// recomputed by the definition, with IEEE divisions, after the tile's main
// loop; the out-of-line exact path then costs the main loop one predicated
// shared atomic. Blocks with eff == 0 (the zero-block guard: all-zero blocks,
// or a zero global scale) fail the same range test and get their sign-kept
// zero codes on the exact path too. Products below the normal range are far below the first
// midpoint and overflowing products far above the last, so neither can change
// a code.
//
// Passes: the tensor amax must be known before any block can be quantized,
// so a first kernel reduces |x| into per-CTA partial maxima (workspace), and
// the block kernel reduces those partials itself (a few KB per CTA, from L2)
// before its first block. The block kernel walks the tiles in reverse order,
// so its first reads hit the tail of the tensor that the amax pass left in
// the 126 MB L2.
//
// Work split of the block pass: a lane owns one block (16 elements, one
// 256-bit load of bf16), writes 8 packed bytes and one scale byte, so a warp
// reads 1 KiB and writes 256 + 32 contiguous bytes per step.
#include <cuda.h>

#include "common.cuh"

namespace mxq {
namespace {

constexpr int kMaxPartials = 2048;  // CTAs of the amax pass (workspace floats)
constexpr int kAmaxSteps = 2;       // 16-element bf16 chunks per thread per iteration (fp32: 1)
constexpr int kAmaxCtasPerSm = 8;   // one resident wave: grid = SMs x 8
constexpr int kSteps = 4;
constexpr int kBlocksPerWarp = 32 * kSteps;
constexpr int kBlocksPerTile = kBlocksPerWarp * (kThreads / 32);
constexpr int kDqSteps = 2;  // dequantize: blocks per lane
constexpr int kDqBlocksPerWarp = 32 * kDqSteps;
constexpr int kDqBlocksPerTile = kDqBlocksPerWarp * (kThreads / 32);

enum GMode { kFromPartials = 0, kGiven = 1, kFromAmax = 2 };

__device__ __forceinline__ float decode_e4m3(uint32_t code) {
  return f16x2_to_f32x2(cvt_f16x2_from_e4m3x2(code)).x;
}

// Reciprocal by the hardware approximation (<= 1 ulp for normal inputs).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// True when |v| in [2^-125, 2^125): its approximate reciprocal is normal.
__device__ __forceinline__ bool rcp_safe(float v) {
  const uint32_t e = __float_as_uint(v) & 0x7f800000u;
  return e >= (2u << 23) && e < (252u << 23);
}

// Distance-like key of v to the nearest value whose mantissa is zero below
// bit `bits`: small (<= 64) when v is within 32 ulps of such a value.
template <int BITS>
__device__ __forceinline__ uint32_t grid_key(float v) {
  return (__float_as_uint(v) + 32u) & ((1u << BITS) - 1u);
}

inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// ------------------------------------------------------------- amax pass

// max |x| over the non-NaN elements of 16-element chunks [c0, c1) (chunk c
// = row c / cpr, columns 16 (c % cpr) ..), taken by CTA j of `ctas` CTAs that
// share the range; 0 for a thread with no chunk.
template <typename InT, bool V8, bool STRIDED>
__device__ __forceinline__ float amax_chunks(const InT* __restrict__ x, uint64_t c0, uint64_t c1,
                                             uint64_t j, uint64_t ctas, uint32_t cpr,
                                             FastDiv rowdiv, int64_t ld) {
  constexpr int steps = sizeof(InT) == 2 ? kAmaxSteps : 1;  // 64 bytes in flight per thread
  float m = 0.0f;
  const uint64_t per_iter = ctas * kThreads * steps;
  for (uint64_t base = c0 + j * kThreads * steps; base < c1; base += per_iter) {
    In16<InT> v[steps];
#pragma unroll
    for (int u = 0; u < steps; u++) {
      const uint64_t c = base + uint64_t(u) * kThreads + threadIdx.x;
      if (c < c1) {
        uint64_t off;
        if constexpr (STRIDED) {
          const uint64_t r = rowdiv.div(c);
          off = r * uint64_t(ld) + (c - r * cpr) * 16;
        } else {
          off = c * 16;
        }
        v[u].template load<V8>(x + off);
      } else {
        v[u].zero();
      }
    }
#pragma unroll
    for (int u = 0; u < steps; u++) m = fmaxf(m, v[u].absmax());
  }
  return m;
}

template <typename InT, bool V8, bool STRIDED>
__global__ void __launch_bounds__(kThreads, kAmaxCtasPerSm)
nvfp4_amax_kernel(const InT* __restrict__ x, uint64_t nchunks, uint32_t cpr, FastDiv rowdiv,
                  int64_t ld, float* __restrict__ partials) {
  pdl_enter();
  __shared__ float red[kThreads / 32];
  float m = amax_chunks<InT, V8, STRIDED>(x, 0, nchunks, blockIdx.x, gridDim.x, cpr, rowdiv, ld);
  m = block_max(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// One CTA: max over the partials into *amax.
__global__ void __launch_bounds__(kThreads)
nvfp4_amax_finalize_kernel(const float* __restrict__ partials, uint32_t n, float* amax) {
  pdl_enter();
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

// Sign-kept zero codes of a block (zero-block guard, eff == 0).
template <typename InT>
__device__ __forceinline__ uint2 zero_codes(const In16<InT>& v) {
  const uint32_t sg = v.signs();
  uint32_t w0 = 0, w1 = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    w0 |= ((sg >> i) & 1u) << (4 * i + 3);
    w1 |= ((sg >> (i + 8)) & 1u) << (4 * i + 3);
  }
  return make_uint2(w0, w1);
}

// Scale byte and codes of one block by the definition, with IEEE divisions:
// the path for the rare blocks whose fast-path decision is not certain. Out
// of line and run after the tile's main loop, so that it costs the main loop
// nothing.
template <typename InT>
__device__ __noinline__ void exact_block(const InT* p, float g, uint8_t* pk, uint8_t* sc) {
  In16<InT> v;
  v.template load<false>(p);
  const float amax = fmaxf(v.absmax(), 0.0f);
  uint32_t sb = 0;
  float eff = 0.0f;
  if (g != 0.0f) {
    sb = cvt_e4m3x2(__fdiv_rn(amax, __fmul_rn(6.0f, g)), 0.0f) & 0xffu;
    eff = __fmul_rn(decode_e4m3(sb), g);
  }
  uint2 codes;
  if (eff == 0.0f) {
    codes = zero_codes(v);
  } else {
    uint32_t b[8];
#pragma unroll
    for (int k = 0; k < 8; k++) b[k] = cvt_e2m1x2(__fdiv_rn(v.lo(k), eff), __fdiv_rn(v.hi(k), eff));
    codes = make_uint2(b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24),
                       b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24));
  }
  st_v2(pk, codes);
  st_u8(sc, sb);
}

// Packed E2M1 codes (8 bytes, element 2k in the low nibble of byte k) of a
// block for eff != 0, from the bracketing products x * r (1 -+ 2^-20); *sure
// is cleared when the two brackets disagree anywhere or eff is outside the
// range where the approximate reciprocal is normal.
template <typename InT>
__device__ __forceinline__ uint2 e2m1_codes(const In16<InT>& v, float eff, bool& sure) {
  const float r = rcp_approx(eff);
  const float rl = __fmul_rn(r, 0.99999904632568359375f);  // 1 - 2^-20
  const float rh = __fmul_rn(r, 1.00000095367431640625f);  // 1 + 2^-20
  float2 l[8], h[8];
#pragma unroll
  for (int k = 0; k < 8; k++) {
    l[k] = mul2(v.lo(k), v.hi(k), rl);
    h[k] = mul2(v.lo(k), v.hi(k), rh);
  }
  const uint2 L = make_uint2(cvt_e2m1x8(l[0], l[1], l[2], l[3]), cvt_e2m1x8(l[4], l[5], l[6], l[7]));
  const uint2 H = make_uint2(cvt_e2m1x8(h[0], h[1], h[2], h[3]), cvt_e2m1x8(h[4], h[5], h[6], h[7]));
  // a code boundary inside some bracket (exact quotients such as 3.5 are
  // common with bf16 inputs) leaves the block to the exact path
  sure = rcp_safe(eff) && ((L.x ^ H.x) | (L.y ^ H.y)) == 0u;
  return L;
}

// Quantizes the tile of blocks [tb0, tb0 + nt) (block = 16 elements, row-
// major over the [M, N] view): all loads are issued first, then get_g()
// supplies the global scale (it may reduce partial maxima meanwhile; every
// thread of the CTA calls it), then scales and codes are written.
template <typename InT, bool V8, bool STRIDED, typename GetG>
__device__ __forceinline__ void quant_tile(const QuantArgs& a, uint64_t tb0, uint32_t nt,
                                           GetG get_g) {
  __shared__ uint16_t fix_list[kBlocksPerTile];  // tile-local blocks for the exact path
  __shared__ uint32_t fix_count[1];
  if (threadIdx.x == 0) *fix_count = 0;
  __syncthreads();
  const bool full = nt == kBlocksPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lb0 = warp * kBlocksPerWarp + lane;
  const InT* x = static_cast<const InT*>(a.x);

  In16<InT> v[kSteps];
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lb = lb0 + 32 * u;
    const InT* p;
    if constexpr (STRIDED) {
      const uint64_t blk = tb0 + lb;
      const uint64_t r = a.rowdiv.div(blk);
      p = x + r * uint64_t(a.ld) + (blk - r * a.bpr) * 16;
    } else {
      p = x + (tb0 + lb) * 16;
    }
    if (full || lb < nt) v[u].template load<V8>(p); else v[u].zero();
  }

  const float g = get_g();
  const bool gzero = (g == 0.0f);
  const float t = __fmul_rn(6.0f, g);
  const bool t_ok = rcp_safe(t);
  const float rt = rcp_approx(t);

  uint8_t* pk = a.packed + tb0 * 8;
  uint8_t* sc = a.bscale + tb0;
#pragma unroll
  for (int u = 0; u < kSteps; u++) {
    const uint32_t lb = lb0 + 32 * u;
    if (!(full || lb < nt)) continue;
    const float amax = fmaxf(v[u].absmax(), 0.0f);  // a block holding only NaNs has amax 0
    uint32_t sb = 0;
    float eff = 0.0f;
    bool sure = true;
    if (!gzero) {
      // E4M3 code of fl(amax / t); the approximate quotient decides unless it
      // is within 32 ulps of a value with four significant bits
      const float s = __fmul_rn(amax, rt);
      sure = t_ok && grid_key<19>(s) > 64u;
      sb = cvt_e4m3x2(s, 0.0f) & 0xffu;  // NaN -> 0x7F
      eff = __fmul_rn(decode_e4m3(sb), g);
    }
    // eff == 0 (the zero-block guard) fails the reciprocal's range test
    // inside e2m1_codes, so such blocks are left to the exact path, which
    // writes their sign-kept zeros; the main loop carries no code for them
    bool sure_codes;
    const uint2 codes = e2m1_codes(v[u], eff, sure_codes);
    sure = sure && sure_codes;
    st_v2(pk + lb * 8, codes);
    st_u8(sc + lb, sb);
    if (__builtin_expect(!sure, 0)) fix_list[atomicAdd(fix_count, 1u)] = uint16_t(lb);
  }

  // the blocks left undecided, by the definition (their input is read again)
  __syncthreads();
  const uint32_t nfix = *fix_count;
  for (uint32_t i = threadIdx.x; i < nfix; i += kThreads) {
    const uint32_t lb = fix_list[i];
    const InT* p;
    if constexpr (STRIDED) {
      const uint64_t blk = tb0 + lb;
      const uint64_t r = a.rowdiv.div(blk);
      p = x + r * uint64_t(a.ld) + (blk - r * a.bpr) * 16;
    } else {
      p = x + (tb0 + lb) * 16;
    }
    exact_block(p, g, pk + lb * 8, sc + lb);
  }
}

template <typename InT, bool V8, bool STRIDED, int GMODE>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_kernel(const __grid_constant__ QuantArgs a) {
  pdl_enter();
  __shared__ float red[kThreads / 32];
  const uint32_t tile = a.ntiles - 1 - blockIdx.x;
  const uint64_t tb0 = uint64_t(tile) * kBlocksPerTile;
  const uint64_t left = a.nblocks - tb0;
  const uint32_t nt = left < kBlocksPerTile ? uint32_t(left) : uint32_t(kBlocksPerTile);
  quant_tile<InT, V8, STRIDED>(a, tb0, nt, [&]() {
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
    return g;
  });
}

// ------------------------------------------------ per-slice global scales

// A tensor cut into S consecutive row ranges ("slices"), each with its own
// global scale. Block (= amax chunk) ranges, amax-pass CTAs and quant tiles
// are assigned per slice, so no CTA spans two slices.
template <int MAXS>
struct SliceTable {
  int32_t S;
  uint64_t bbase[MAXS + 1];  // first block of slice s; bbase[S] = all blocks
  uint32_t cbase[MAXS + 1];  // first amax-pass CTA (= partial) of slice s
  uint32_t tbase[MAXS + 1];  // first quant tile of slice s
};

// The slice whose range [base[s], base[s+1]) holds v (v < base[S]).
__device__ __forceinline__ int find_slice(const uint32_t* base, int S, uint32_t v) {
  int lo = 0, hi = S;  // invariant: base[lo] <= v < base[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (base[mid] <= v) lo = mid; else hi = mid;
  }
  return lo;
}

template <typename InT, bool V8, bool STRIDED, int MAXS>
__global__ void __launch_bounds__(kThreads, kAmaxCtasPerSm)
nvfp4_amax_sliced_kernel(const InT* __restrict__ x, uint32_t cpr, FastDiv rowdiv, int64_t ld,
                         float* __restrict__ partials, const __grid_constant__ SliceTable<MAXS> t) {
  pdl_enter();
  __shared__ float red[kThreads / 32];
  const int s = find_slice(t.cbase, t.S, blockIdx.x);
  float m = amax_chunks<InT, V8, STRIDED>(x, t.bbase[s], t.bbase[s + 1], blockIdx.x - t.cbase[s],
                                          t.cbase[s + 1] - t.cbase[s], cpr, rowdiv, ld);
  m = block_max(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// One warp per slice: max over the slice's partials into amax[s] (0 for an
// empty slice).
template <int MAXS>
__global__ void __launch_bounds__(kThreads)
nvfp4_amax_sliced_finalize_kernel(const float* __restrict__ partials, float* __restrict__ amax,
                                  const __grid_constant__ SliceTable<MAXS> t) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int s = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  if (s >= t.S) return;
  float m = 0.0f;
  for (uint32_t i = t.cbase[s] + lane; i < t.cbase[s + 1]; i += 32) m = fmaxf(m, partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  if (lane == 0) amax[s] = m;
}

template <typename InT, bool V8, bool STRIDED, int GMODE, int MAXS>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_sliced_kernel(const __grid_constant__ QuantArgs a,
                          const __grid_constant__ SliceTable<MAXS> t) {
  pdl_enter();
  __shared__ float red[kThreads / 32];
  if constexpr (GMODE != kGiven) {
    // global scales of empty slices (no tile of theirs runs)
    if (blockIdx.x == 0) {
      for (int e = threadIdx.x; e < t.S; e += kThreads) {
        if (t.bbase[e] == t.bbase[e + 1]) {
          if constexpr (GMODE == kFromAmax) a.gs[e] = __fdiv_rn(a.amax_in[e], 2688.0f);
          else a.gs[e] = 0.0f;
        }
      }
    }
  }
  const uint32_t tile = a.ntiles - 1 - blockIdx.x;
  const int s = find_slice(t.tbase, t.S, tile);
  const uint64_t tb0 = t.bbase[s] + uint64_t(tile - t.tbase[s]) * kBlocksPerTile;
  const uint64_t left = t.bbase[s + 1] - tb0;
  const uint32_t nt = left < kBlocksPerTile ? uint32_t(left) : uint32_t(kBlocksPerTile);
  quant_tile<InT, V8, STRIDED>(a, tb0, nt, [&]() {
    float g;
    if constexpr (GMODE == kGiven) {
      g = a.gs[s];
    } else {
      float A;
      if constexpr (GMODE == kFromAmax) {
        A = a.amax_in[s];
      } else {
        float m = 0.0f;
        for (uint32_t i = t.cbase[s] + threadIdx.x; i < t.cbase[s + 1]; i += kThreads)
          m = fmaxf(m, a.partials[i]);
        A = block_max(m, red);
      }
      g = __fdiv_rn(A, 2688.0f);
      if (tile == t.tbase[s] && threadIdx.x == 0) a.gs[s] = g;
    }
    return g;
  });
}

// --------------------------------------------------------------- dequant

template <typename OutT, bool V8>
__global__ void __launch_bounds__(kThreads)
nvfp4_dequant_kernel(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ bscale,
                     const float* __restrict__ gs, OutT* __restrict__ y, uint64_t nblocks) {
  pdl_enter();
  const uint64_t tb0 = uint64_t(blockIdx.x) * kDqBlocksPerTile;
  const uint64_t left = nblocks - tb0;
  const uint32_t nt = left < kDqBlocksPerTile ? uint32_t(left) : uint32_t(kDqBlocksPerTile);
  const bool full = nt == kDqBlocksPerTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lb0 = warp * kDqBlocksPerWarp + lane;
  uint2 w[kDqSteps];
  uint32_t sb[kDqSteps];
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lb = lb0 + 32 * u;
    if (full || lb < nt) {
      w[u] = ld_nc_v2(packed + (tb0 + lb) * 8);
      sb[u] = ld_nc_u8(bscale + tb0 + lb);
    } else {
      w[u] = make_uint2(0, 0);
      sb[u] = 0;
    }
  }
  const float g = *gs;
#pragma unroll
  for (int u = 0; u < kDqSteps; u++) {
    const uint32_t lb = lb0 + 32 * u;
    if (!(full || lb < nt)) continue;
    const float eff = __fmul_rn(decode_e4m3(sb[u]), g);
    float f[16];
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const uint32_t byte = ((k < 4 ? w[u].x : w[u].y) >> (8 * (k & 3))) & 0xffu;
      const float2 d = f16x2_to_f32x2(cvt_f16x2_from_e2m1x2(byte));
      const float2 p = mul2(d.x, d.y, eff);
      f[2 * k] = p.x;
      f[2 * k + 1] = p.y;
    }
    if (!isfinite(eff)) {  // only then can a product be NaN (0 * inf, NaN scale)
#pragma unroll
      for (int i = 0; i < 16; i++)
        if (isnan(f[i])) f[i] = __uint_as_float(0x7fc00000u);
    }
    OutT* dst = y + (tb0 + lb) * 16;
    if constexpr (sizeof(OutT) == 2) {
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 8; k++) o[k] = cvt_bf16x2(f[2 * k], f[2 * k + 1]);
      if (!isfinite(eff)) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
          if (isnan(f[i])) {
            const int sh = 16 * (i & 1);
            o[i >> 1] = (o[i >> 1] & ~(0xffffu << sh)) | (0x7fc0u << sh);
          }
        }
      }
      if constexpr (V8) {
        st_v8(dst, o);
      } else {
        st_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
        st_v4(dst + 8, make_uint4(o[4], o[5], o[6], o[7]));
      }
    } else {
      uint32_t o[16];
#pragma unroll
      for (int i = 0; i < 16; i++) o[i] = __float_as_uint(f[i]);
      if constexpr (V8) {
        st_v8(dst, *reinterpret_cast<const uint32_t(*)[8]>(&o[0]));
        st_v8(dst + 8, *reinterpret_cast<const uint32_t(*)[8]>(&o[8]));
      } else {
#pragma unroll
        for (int i = 0; i < 4; i++)
          st_v4(dst + 4 * i, make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
      }
    }
  }
}

// ------------------------------------------------------------------ host


template <typename InT, bool V8, bool STRIDED>
cudaError_t launch_amax_kernel(uint32_t grid, const void* x, uint64_t nchunks, uint32_t cpr,
                               FastDiv rd, int64_t ld, float* partials, cudaStream_t s) {
  return launch_pdl(nvfp4_amax_kernel<InT, V8, STRIDED>, grid, s, static_cast<const InT*>(x),
                    nchunks, cpr, rd, ld, partials);
}

// Launches the amax pass into `partials`; returns the number of partials.
mxq_status launch_amax(const void* x, int dt, int64_t M, int64_t N, int64_t ld, float* partials,
                       uint32_t* npartials, cudaStream_t s) {
  const uint64_t cpr = uint64_t(N) / 16;
  const uint64_t nchunks = uint64_t(M) * cpr;
  const uint64_t per_cta = uint64_t(kThreads) * kAmaxSteps;
  uint64_t grid = (nchunks + per_cta - 1) / per_cta;
  const uint64_t cap = std::min<uint64_t>(kMaxPartials, uint64_t(sm_count()) * kAmaxCtasPerSm);
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const FastDiv rd = FastDiv::make(uint32_t(cpr));
  const bool strided = ld != N;
  const bool v8 = aligned32(x) && (uint64_t(ld) * elem_size(dt)) % 32 == 0;
  const uint32_t G = uint32_t(grid);
#define MXQ_AMAX(T, V, S) e = launch_amax_kernel<T, V, S>(G, x, nchunks, uint32_t(cpr), rd, ld, partials, s)
  cudaError_t e;
  if (dt == MXQ_BF16) {
    if (v8) { if (strided) MXQ_AMAX(uint16_t, true, true); else MXQ_AMAX(uint16_t, true, false); }
    else { if (strided) MXQ_AMAX(uint16_t, false, true); else MXQ_AMAX(uint16_t, false, false); }
  } else {
    if (v8) { if (strided) MXQ_AMAX(float, true, true); else MXQ_AMAX(float, true, false); }
    else { if (strided) MXQ_AMAX(float, false, true); else MXQ_AMAX(float, false, false); }
  }
#undef MXQ_AMAX
  *npartials = G;
  return launched(e);
}

template <typename InT, bool V8, bool STRIDED>
mxq_status launch_quant_mode(const QuantArgs& a, int mode, cudaStream_t s) {
  switch (mode) {
    case kGiven:
      return launched(launch_pdl(nvfp4_quant_kernel<InT, V8, STRIDED, kGiven>, a.ntiles, s, a));
    case kFromAmax:
      return launched(launch_pdl(nvfp4_quant_kernel<InT, V8, STRIDED, kFromAmax>, a.ntiles, s, a));
    default:
      return launched(launch_pdl(nvfp4_quant_kernel<InT, V8, STRIDED, kFromPartials>, a.ntiles, s, a));
  }
}

template <typename InT>
mxq_status launch_quant_typed(const QuantArgs& a, int mode, bool v8, bool strided, cudaStream_t s) {
  if (v8) return strided ? launch_quant_mode<InT, true, true>(a, mode, s)
                         : launch_quant_mode<InT, true, false>(a, mode, s);
  return strided ? launch_quant_mode<InT, false, true>(a, mode, s)
                 : launch_quant_mode<InT, false, false>(a, mode, s);
}

mxq_status check_input(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x) {
  if (!valid_dtype(dt)) return MXQ_ERR_DTYPE;
  if (M < 0 || N < 0 || N % 16 != 0 || ld_x < N) return MXQ_ERR_SHAPE;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!x) return MXQ_ERR_NULL;
  const uint64_t nblocks = uint64_t(M) * (uint64_t(N) / 16);
  if (uint64_t(N) / 16 > 0xffffffffull || (nblocks + kBlocksPerTile - 1) / kBlocksPerTile > 0x7fffffffull)
    return MXQ_ERR_SHAPE;
  if (!aligned16(x) || (uint64_t(ld_x) * elem_size(dt)) % 16 != 0) return MXQ_ERR_ALIGN;
  return MXQ_OK;
}

// ------------------------------------------------------- sliced (host)

mxq_status check_slices(int32_t S, const int64_t* rows, int64_t M) {
  if (S < 1 || S > MXQ_NVFP4_MAX_SLICES) return MXQ_ERR_SHAPE;
  if (!rows) return MXQ_ERR_NULL;
  int64_t total = 0;
  for (int32_t s = 0; s < S; s++) {
    if (rows[s] < 0 || rows[s] > M - total) return MXQ_ERR_SHAPE;
    total += rows[s];
  }
  return total == M ? MXQ_OK : MXQ_ERR_SHAPE;
}

// Block, amax-CTA and tile ranges per slice. The amax pass gets about
// min(2048, SMs x 8) CTAs in all, shared out in proportion to the slices'
// sizes, at least one per non-empty slice (so at most 2048 + S partials).
template <int MAXS>
mxq_status build_slices(int32_t S, const int64_t* rows, int64_t N, SliceTable<MAXS>& t) {
  const uint64_t bpr = uint64_t(N) / 16;
  uint64_t total = 0;
  for (int32_t s = 0; s < S; s++) total += uint64_t(rows[s]) * bpr;
  const uint64_t per_cta = uint64_t(kThreads) * kAmaxSteps;
  const uint64_t K = std::min<uint64_t>(kMaxPartials, uint64_t(sm_count()) * kAmaxCtasPerSm);
  uint64_t b = 0, c = 0, tl = 0;
  t.S = S;
  for (int32_t s = 0; s < S; s++) {
    t.bbase[s] = b;
    t.cbase[s] = uint32_t(c);
    t.tbase[s] = uint32_t(tl);
    const uint64_t n = uint64_t(rows[s]) * bpr;
    if (n) {
      uint64_t cs = uint64_t((unsigned __int128)K * n / total);
      const uint64_t need = (n + per_cta - 1) / per_cta;
      cs = cs > need ? need : cs;
      c += cs < 1 ? 1 : cs;
    }
    tl += (n + kBlocksPerTile - 1) / kBlocksPerTile;
    b += n;
    if (tl > 0x7fffffffull) return MXQ_ERR_SHAPE;
  }
  t.bbase[S] = b;
  t.cbase[S] = uint32_t(c);
  t.tbase[S] = uint32_t(tl);
  return MXQ_OK;
}

template <typename InT, bool V8, bool STRIDED, int MAXS>
cudaError_t launch_amax_sliced_kernel(const void* x, uint32_t cpr, FastDiv rd, int64_t ld,
                                      float* partials, const SliceTable<MAXS>& t, cudaStream_t s) {
  return launch_pdl(nvfp4_amax_sliced_kernel<InT, V8, STRIDED, MAXS>, t.cbase[t.S], s,
                    static_cast<const InT*>(x), cpr, rd, ld, partials, t);
}

template <int MAXS>
mxq_status launch_amax_sliced(const void* x, int dt, int64_t N, int64_t ld, float* partials,
                              const SliceTable<MAXS>& t, cudaStream_t s) {
  const uint32_t cpr = uint32_t(uint64_t(N) / 16);
  const FastDiv rd = FastDiv::make(cpr);
  const bool strided = ld != N;
  const bool v8 = aligned32(x) && (uint64_t(ld) * elem_size(dt)) % 32 == 0;
#define MXQ_AMAX_S(T, V, S) e = launch_amax_sliced_kernel<T, V, S, MAXS>(x, cpr, rd, ld, partials, t, s)
  cudaError_t e;
  if (dt == MXQ_BF16) {
    if (v8) { if (strided) MXQ_AMAX_S(uint16_t, true, true); else MXQ_AMAX_S(uint16_t, true, false); }
    else { if (strided) MXQ_AMAX_S(uint16_t, false, true); else MXQ_AMAX_S(uint16_t, false, false); }
  } else {
    if (v8) { if (strided) MXQ_AMAX_S(float, true, true); else MXQ_AMAX_S(float, true, false); }
    else { if (strided) MXQ_AMAX_S(float, false, true); else MXQ_AMAX_S(float, false, false); }
  }
#undef MXQ_AMAX_S
  return launched(e);
}

template <typename InT, bool V8, bool STRIDED, int MAXS>
mxq_status launch_quant_sliced_mode(const QuantArgs& a, const SliceTable<MAXS>& t, int mode,
                                    cudaStream_t s) {
  switch (mode) {
    case kGiven:
      return launched(launch_pdl(nvfp4_quant_sliced_kernel<InT, V8, STRIDED, kGiven, MAXS>, a.ntiles, s, a, t));
    case kFromAmax:
      return launched(launch_pdl(nvfp4_quant_sliced_kernel<InT, V8, STRIDED, kFromAmax, MAXS>, a.ntiles, s, a, t));
    default:
      return launched(launch_pdl(nvfp4_quant_sliced_kernel<InT, V8, STRIDED, kFromPartials, MAXS>, a.ntiles, s, a, t));
  }
}

template <typename InT, int MAXS>
mxq_status launch_quant_sliced_typed(const QuantArgs& a, const SliceTable<MAXS>& t, int mode,
                                     bool v8, bool strided, cudaStream_t s) {
  if (v8) return strided ? launch_quant_sliced_mode<InT, true, true, MAXS>(a, t, mode, s)
                         : launch_quant_sliced_mode<InT, true, false, MAXS>(a, t, mode, s);
  return strided ? launch_quant_sliced_mode<InT, false, true, MAXS>(a, t, mode, s)
                 : launch_quant_sliced_mode<InT, false, false, MAXS>(a, t, mode, s);
}

template <int MAXS>
mxq_status amax_sliced_impl(const void* x, int dt, int64_t N, int64_t ld_x, int32_t S,
                            const int64_t* rows, float* amax, float* partials, cudaStream_t s) {
  SliceTable<MAXS> t;
  mxq_status st = build_slices<MAXS>(S, rows, N, t);
  if (st != MXQ_OK) return st;
  st = launch_amax_sliced<MAXS>(x, dt, N, ld_x, partials, t, s);
  if (st != MXQ_OK) return st;
  const uint32_t grid = uint32_t((S + kThreads / 32 - 1) / (kThreads / 32));
  return launched(launch_pdl(nvfp4_amax_sliced_finalize_kernel<MAXS>, grid, s,
                             static_cast<const float*>(partials), amax, t));
}

template <int MAXS>
mxq_status quantize_sliced_impl(QuantArgs& a, int dt, int64_t N, int64_t ld_x, int32_t S,
                                const int64_t* rows, int mode, float* partials, cudaStream_t s) {
  SliceTable<MAXS> t;
  mxq_status st = build_slices<MAXS>(S, rows, N, t);
  if (st != MXQ_OK) return st;
  a.ntiles = t.tbase[S];
  if (mode == kFromPartials) {
    a.partials = partials;
    st = launch_amax_sliced<MAXS>(a.x, dt, N, ld_x, partials, t, s);
    if (st != MXQ_OK) return st;
  }
  const bool strided = ld_x != N;
  const bool v8 = aligned32(a.x) && (uint64_t(ld_x) * elem_size(dt)) % 32 == 0;
  if (dt == MXQ_BF16) return launch_quant_sliced_typed<uint16_t, MAXS>(a, t, mode, v8, strided, s);
  return launch_quant_sliced_typed<float, MAXS>(a, t, mode, v8, strided, s);
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
  return launched(launch_pdl(nvfp4_amax_finalize_kernel, 1, s,
                             static_cast<const float*>(workspace), np, amax));
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
  const int mode = given ? kGiven : (amax_in ? kFromAmax : kFromPartials);
  if (pass1) {
    a.partials = static_cast<const float*>(workspace);
    st = launch_amax(x, dt, M, N, ld_x, static_cast<float*>(workspace), &a.npartials, s);
    if (st != MXQ_OK) return st;
  }
  const bool strided = ld_x != N;
  const bool v8 = aligned32(x) && (uint64_t(ld_x) * elem_size(dt)) % 32 == 0;
  if (dt == MXQ_BF16) return launch_quant_typed<uint16_t>(a, mode, v8, strided, s);
  return launch_quant_typed<float>(a, mode, v8, strided, s);
}

size_t mxq_nvfp4_sliced_workspace_bytes(int32_t n_slices) {
  if (n_slices < 1 || n_slices > MXQ_NVFP4_MAX_SLICES) return 0;
  return sizeof(float) * (size_t(mxq::kMaxPartials) + size_t(n_slices));
}

mxq_status nvfp4_amax_sliced(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                             int32_t n_slices, const int64_t* slice_rows, float* amax,
                             void* workspace, size_t ws_bytes, mxq_stream_t stream) {
  using namespace mxq;
  mxq_status st = check_input(x, dt, M, N, ld_x);
  if (st != MXQ_OK) return st;
  st = check_slices(n_slices, slice_rows, M);
  if (st != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!amax) return MXQ_ERR_NULL;
  if (!workspace || ws_bytes < mxq_nvfp4_sliced_workspace_bytes(n_slices) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3u))
    return MXQ_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partials = static_cast<float*>(workspace);
  if (n_slices <= 64)
    return amax_sliced_impl<64>(x, dt, N, ld_x, n_slices, slice_rows, amax, partials, s);
  return amax_sliced_impl<MXQ_NVFP4_MAX_SLICES>(x, dt, N, ld_x, n_slices, slice_rows, amax,
                                                 partials, s);
}

mxq_status nvfp4_quantize_sliced(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                                 int32_t n_slices, const int64_t* slice_rows, uint8_t* packed,
                                 uint8_t* block_scale, float* global_scales,
                                 const float* amax_in, uint32_t flags, void* workspace,
                                 size_t ws_bytes, mxq_stream_t stream) {
  using namespace mxq;
  if (flags & ~MXQ_NVFP4_GLOBAL_GIVEN) return MXQ_ERR_ARG;
  const bool given = (flags & MXQ_NVFP4_GLOBAL_GIVEN) != 0;
  if (given && amax_in) return MXQ_ERR_ARG;
  mxq_status st = check_input(x, dt, M, N, ld_x);
  if (st != MXQ_OK) return st;
  st = check_slices(n_slices, slice_rows, M);
  if (st != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!packed || !block_scale || !global_scales) return MXQ_ERR_NULL;
  if (!aligned16(packed)) return MXQ_ERR_ALIGN;
  const bool pass1 = !given && !amax_in;
  if (pass1 && (!workspace || ws_bytes < mxq_nvfp4_sliced_workspace_bytes(n_slices) ||
                (reinterpret_cast<uintptr_t>(workspace) & 3u)))
    return MXQ_ERR_WORKSPACE;
  QuantArgs a{};
  a.x = x;
  a.ld = ld_x;
  a.bpr = uint32_t(uint64_t(N) / 16);
  a.rowdiv = FastDiv::make(a.bpr);
  a.packed = packed;
  a.bscale = block_scale;
  a.gs = global_scales;
  a.amax_in = amax_in;
  a.nblocks = uint64_t(M) * a.bpr;
  const int mode = given ? kGiven : (amax_in ? kFromAmax : kFromPartials);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partials = static_cast<float*>(workspace);
  if (n_slices <= 64)
    return quantize_sliced_impl<64>(a, dt, N, ld_x, n_slices, slice_rows, mode, partials, s);
  return quantize_sliced_impl<MXQ_NVFP4_MAX_SLICES>(a, dt, N, ld_x, n_slices, slice_rows, mode,
                                                     partials, s);
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
  const uint64_t tiles = (nblocks + kDqBlocksPerTile - 1) / kDqBlocksPerTile;
  if (tiles > 0x7fffffffull) return MXQ_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t grid = uint32_t(tiles);
  const bool v8 = aligned32(y);
  if (out_dt == MXQ_BF16) {
    uint16_t* yp = static_cast<uint16_t*>(y);
    return launched(v8 ? launch_pdl(nvfp4_dequant_kernel<uint16_t, true>, grid, s, packed, block_scale, global_scale, yp, nblocks)
                       : launch_pdl(nvfp4_dequant_kernel<uint16_t, false>, grid, s, packed, block_scale, global_scale, yp, nblocks));
  }
  float* yp = static_cast<float*>(y);
  return launched(v8 ? launch_pdl(nvfp4_dequant_kernel<float, true>, grid, s, packed, block_scale, global_scale, yp, nblocks)
                     : launch_pdl(nvfp4_dequant_kernel<float, false>, grid, s, packed, block_scale, global_scale, yp, nblocks));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// nvfp4_quantize_noalloc: the same quantization for callers that cannot
// allocate device memory when they quantize, e.g. code that runs inside a
// serving engine or plugin with a fixed, pre-planned memory budget, or a C
// program with no device allocator at hand. Its only scratch (the per-CTA
// partial maxima of the tensor-amax pass) lives in the fixed array below,
// which every GPU that loads this library holds until the process exits.

namespace mxq {
namespace {

constexpr int kNoallocPartials = kMaxPartials;  // 2048 floats = 8 KiB per device
static __device__ __align__(256) float g_noalloc_partials[kNoallocPartials];

constexpr int kMaxDevices = 256;

// The array's device address is cached per device together with the id of
// the CUDA context it was looked up in. A context that is destroyed and
// created again (cudaDeviceReset, or a driver-API context of the caller's)
// reloads the library's module, and the array may then sit elsewhere: a
// changed context id makes the next call look the address up again.
struct NoallocSlot {
  unsigned long long ctx_id;  // 0: nothing cached
  float* ptr;
};
std::mutex g_noalloc_mu;
NoallocSlot g_noalloc_slot[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current CUDA context (driver entry points
// fetched through the runtime, so the library needs no link against the
// driver library); false when there is none yet or the driver lacks the call.
bool current_context_id(unsigned long long* id) {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

// Device address of g_noalloc_partials in the current device's context. The
// first call on a device (and the first after that device's context changed)
// looks it up with cudaGetSymbolAddress, with that device current; later
// calls reuse it. Without a context id to key on, every call looks it up.
mxq_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MXQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MXQ_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  unsigned long long id = 0;
  if (slot.ptr != nullptr && current_context_id(&id) && id == slot.ctx_id) {
    *out = slot.ptr;
    return MXQ_OK;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_partials);
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MXQ_ERR_CUDA;
  }
  // the lookup made the device's context current if it was not yet
  slot.ptr = current_context_id(&id) ? static_cast<float*>(p) : nullptr;
  slot.ctx_id = slot.ptr ? id : 0;
  *out = static_cast<float*>(p);
  return MXQ_OK;
}

}  // namespace
}  // namespace mxq

extern "C" mxq_status nvfp4_quantize_noalloc(const void* x, int dt, int64_t M, int64_t N,
                                             int64_t ld_x, uint8_t* packed,
                                             uint8_t* block_scale, float* global_scale,
                                             const float* amax_in, uint32_t flags,
                                             mxq_stream_t stream) {
  using namespace mxq;
  // the same argument checks as nvfp4_quantize, before the one-time set-up
  if (flags & ~MXQ_NVFP4_GLOBAL_GIVEN) return MXQ_ERR_ARG;
  if ((flags & MXQ_NVFP4_GLOBAL_GIVEN) && amax_in) return MXQ_ERR_ARG;
  mxq_status st = check_input(x, dt, M, N, ld_x);
  if (st != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  if (!packed || !block_scale || !global_scale) return MXQ_ERR_NULL;
  if (!aligned16(packed)) return MXQ_ERR_ALIGN;
  // scratch needed by this call versus what the fixed array holds
  const size_t need = mxq_nvfp4_workspace_bytes(M, N);
  if (need > sizeof(float) * kNoallocPartials) return MXQ_ERR_WORKSPACE;
  const bool pass1 = !(flags & MXQ_NVFP4_GLOBAL_GIVEN) && amax_in == nullptr;
  float* scratch = nullptr;
  if (pass1) {
    st = noalloc_scratch(&scratch);
    if (st != MXQ_OK) return st;
  }
  return nvfp4_quantize(x, dt, M, N, ld_x, packed, block_scale, global_scale, amax_in, flags,
                        scratch, scratch ? sizeof(float) * kNoallocPartials : 0, stream);
}
