// common.cuh -- device and host helpers shared by the libmxq kernels (sm_100a).
//
// Numerics: the library is compiled without fast math (-ftz=false,
// -prec-div=true, -fmad=false), so fp32 multiplies and divides are IEEE
// round-to-nearest-even with subnormals kept; the power-of-two scaling of the
// MXFP8 path is therefore exact wherever the E4M3 / E8M0 definitions need it
// to be (see mxfp8.cu).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include "mxq.h"

namespace mxq {

constexpr int kThreads = 256;          // threads per CTA in every kernel
constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------------ host

// Records the message of a failed CUDA call for mxq_last_cuda_error().
void record_cuda_error(cudaError_t e);

// Status after a launch: MXQ_ERR_CUDA (and the message recorded) if the
// launch failed.
mxq_status check_launch();

// Status of a launch call followed by the launch's own error state.
inline mxq_status launched(cudaError_t e) {
  if (e != cudaSuccess) {
    record_cuda_error(e);
    cudaGetLastError();
    return MXQ_ERR_CUDA;
  }
  return check_launch();
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int elem_size(int dt) { return dt == MXQ_BF16 ? 2 : 4; }

inline bool valid_dtype(int dt) { return dt == MXQ_BF16 || dt == MXQ_FP32; }

// n / d for 64-bit n and 32-bit d, as one multiply-high: with
// magic = ceil(2^64 / d), floor(n * magic / 2^64) == floor(n / d) whenever
// n * d < 2^64 (the rounding error n * (magic - 2^64/d) / 2^64 stays below
// 1/d, the smallest possible distance of n/d to the next integer).
struct FastDiv {
  uint64_t magic;
  uint32_t d;

  static FastDiv make(uint32_t div) {
    FastDiv f;
    f.d = div;
    f.magic = (div <= 1) ? 0 : (~0ull / div) + 1;
    return f;
  }
  __device__ __forceinline__ uint64_t div(uint64_t n) const {
    return d == 1 ? n : __umul64hi(n, magic);
  }
};

// ---------------------------------------------------------------- device

// 16-byte read-only load that does not allocate in L1 (streamed once).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  uint2 r;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
  uint32_t r;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_nc_u8(const void* p) {
  uint32_t r;
  asm("ld.global.nc.u8 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_v2(void* p, uint2 v) {
  asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void st_u32(void* p, uint32_t v) {
  asm volatile("st.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_u8(void* p, uint32_t v) {
  asm volatile("st.global.u8 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Elementwise max of two bf16 pairs. PTX max ignores a NaN operand (returns
// the other one), which is the amax rule: NaN never raises the maximum.
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Elementwise max of |a| and |b| for two bf16 pairs (the sign of each result
// half is the xor of the input signs and is masked off by the caller); a NaN
// operand is ignored.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// 32-byte read-only load (sm_100 256-bit global load); p must be 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&w)[8]) {
  asm("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
        "=r"(w[7])
      : "l"(p));
}

// 32-byte store (sm_100 256-bit global store); p must be 32-byte aligned.
__device__ __forceinline__ void st_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Two independent IEEE fp32 products (a0*b, a1*b) in one packed instruction
// (sm_100 mul.rn.f32x2; subnormals kept).
__device__ __forceinline__ float2 mul2(float a0, float a1, float b) {
  float2 r;
  asm("{ .reg .b64 a, m, d; mov.b64 a, {%2, %3}; mov.b64 m, {%4, %4};\n\t"
      "mul.rn.f32x2 d, a, m; mov.b64 {%0, %1}, d; }"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a0), "f"(a1), "f"(b));
  return r;
}

// fp32 value of the low / high bf16 of a packed pair (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// (x0 * m, x1 * m) for bf16 elements x0 (selected half SA of word a) and x1
// (half SB of word b) and a power of two m whose fp32 bit pattern has a zero
// low half (every MX multiplier 2^(127 - byte), the subnormal 2^-127
// included, is also a bf16). sm_100 mixed-precision fma: the bf16 product is
// formed exactly and rounded once to fp32, which makes it equal to the fp32
// product of the widened operands; the addend is -0 so that a zero product
// keeps its sign. Saves widening each bf16 element first.
template <int SA, int SB>
__device__ __forceinline__ float2 mul_bf16_pow2(uint32_t a, uint32_t b, float m) {
  const uint32_t mb = __float_as_uint(m) >> 16;
  float r0, r1;
  if constexpr (SA == 0 && SB == 0)
    asm("{ .reg .b16 a0, a1, b0, b1, s, z; mov.b32 {a0, a1}, %2; mov.b32 {b0, b1}, %3;\n\t"
        "mov.b32 {s, z}, %4; fma.rn.f32.bf16 %0, a0, s, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %1, b0, s, 0f80000000; }"
        : "=f"(r0), "=f"(r1) : "r"(a), "r"(b), "r"(mb));
  else if constexpr (SA == 1 && SB == 1)
    asm("{ .reg .b16 a0, a1, b0, b1, s, z; mov.b32 {a0, a1}, %2; mov.b32 {b0, b1}, %3;\n\t"
        "mov.b32 {s, z}, %4; fma.rn.f32.bf16 %0, a1, s, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %1, b1, s, 0f80000000; }"
        : "=f"(r0), "=f"(r1) : "r"(a), "r"(b), "r"(mb));
  else
    asm("{ .reg .b16 a0, a1, b0, b1, s, z; mov.b32 {a0, a1}, %2; mov.b32 {b0, b1}, %3;\n\t"
        "mov.b32 {s, z}, %4; fma.rn.f32.bf16 %0, a0, s, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %1, b1, s, 0f80000000; }"
        : "=f"(r0), "=f"(r1) : "r"(a), "r"(b), "r"(mb));
  return make_float2(r0, r1);
}

// Both bf16 elements of one word times the power of two m (as above).
__device__ __forceinline__ float2 mul_bf16x2_pow2(uint32_t w, float m) {
  return mul_bf16_pow2<0, 1>(w, w, m);
}

// Two fp32 -> E4M3 codes (round to nearest even, |v| > 448 -> 448, NaN ->
// NaN); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (low byte first) -> f16x2 (exact: E4M3 is a subset of f16).
__device__ __forceinline__ uint32_t cvt_f16x2_from_e4m3x2(uint32_t codes) {
  uint32_t r;
  uint16_t c = static_cast<uint16_t>(codes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c));
  return r;
}

// fp32 values of a packed f16 pair (exact).
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h) {
  __half2 v;
  memcpy(&v, &h, 4);
  return __half22float2(v);
}

// Two fp32 -> packed bf16 pair, round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 -> E2M1 codes in one byte (round to nearest even, |u| > 6 -> 6);
// `lo` lands in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Four bytes of E2M1 codes for eight values, two per byte, the first value of
// each pair in the low nibble and pair p in byte p (one register pack, no
// byte shuffles).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float2 p0, float2 p1, float2 p2, float2 p3) {
  uint32_t r;
  asm("{ .reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(r)
      : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
  return r;
}

// One byte holding two E2M1 codes (low nibble first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t cvt_f16x2_from_e2m1x2(uint32_t byte) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "r"(byte));
  return r;
}

// Per-byte flag (0x80) for the E4M3 NaN codes 0x7F / 0xFF in a word of four
// codes. Bytes are at most 0x7F after the mask, so the +1 never carries.
__device__ __forceinline__ uint32_t e4m3_nan_bytes(uint32_t w) {
  return ((w & 0x7f7f7f7fu) + 0x01010101u) & 0x80808080u;
}

// ------------------------------------------------------------ MX scales

// Biased E8M0 exponent of a group's amax (amax >= 0, not NaN) by the OCP MX
// rule for an element format whose largest normal has exponent EMAX (8 for
// E4M3, 2 for E2M1): 127 for amax == 0, 254 for amax == inf, else
// clamp(E(amax) - EMAX, 0, 254) with E the biased fp32 exponent field (the
// same number as floor(log2 amax) + 127 - EMAX, clamped).
template <int EMAX>
__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const uint32_t E = bits >> 23;
  uint32_t b = max(E, uint32_t(EMAX)) - uint32_t(EMAX);
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

// ------------------------------------------------------ 8-element lanes

// Eight consecutive input elements held by one lane: one 16-byte load of
// bf16 bit patterns, or two of fp32.
template <typename InT>
struct In8;

template <>
struct In8<uint16_t> {
  uint32_t w[4];
  __device__ __forceinline__ void load(const uint16_t* p) {
    const uint4 t = ld_nc_v4(p);
    w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
  }
  __device__ __forceinline__ void zero() { w[0] = w[1] = w[2] = w[3] = 0; }
  // max |x| over the non-NaN elements (NaN if all are NaN)
  __device__ __forceinline__ float absmax() const {
    uint32_t m = max_bf16x2(w[0] & 0x7fff7fffu, w[1] & 0x7fff7fffu);
    m = max_bf16x2(m, w[2] & 0x7fff7fffu);
    m = max_bf16x2(m, w[3] & 0x7fff7fffu);
    return fmaxf(bf16_lo(m), bf16_hi(m));
  }
  __device__ __forceinline__ float operator[](int i) const {
    return (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
  }
};

template <>
struct In8<float> {
  uint32_t w[8];
  __device__ __forceinline__ void load(const float* p) {
    const uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 8; i++) w[i] = 0;
  }
  __device__ __forceinline__ float absmax() const {
    float m = fabsf(__uint_as_float(w[0]));
#pragma unroll
    for (int i = 1; i < 8; i++) m = fmaxf(m, fabsf(__uint_as_float(w[i])));
    return m;
  }
  __device__ __forceinline__ float operator[](int i) const { return __uint_as_float(w[i]); }
};

// Sixteen consecutive input elements held by one lane: 32 bytes of bf16 or 64
// of fp32, read with 256-bit loads when V8 (32-byte aligned) or 128-bit ones.
template <typename InT>
struct In16;

template <>
struct In16<uint16_t> {
  uint32_t w[8];
  template <bool V8>
  __device__ __forceinline__ void load(const uint16_t* p) {
    if constexpr (V8) {
      ld_nc_v8(p, w);
    } else {
      const uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + 8);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 8; i++) w[i] = 0;
  }
  // max |x| over the non-NaN elements (NaN if all are NaN)
  __device__ __forceinline__ float absmax() const {
    uint32_t m = absmax_bf16x2(w[0], w[1]);
    const uint32_t m2 = absmax_bf16x2(w[2], w[3]);
    const uint32_t m3 = absmax_bf16x2(w[4], w[5]);
    const uint32_t m4 = absmax_bf16x2(w[6], w[7]);
    m = absmax_bf16x2(absmax_bf16x2(m, m2), absmax_bf16x2(m3, m4)) & 0x7fff7fffu;
    return fmaxf(bf16_lo(m), bf16_hi(m));
  }
  __device__ __forceinline__ float lo(int k) const { return bf16_lo(w[k]); }  // element 2k
  __device__ __forceinline__ float hi(int k) const { return bf16_hi(w[k]); }  // element 2k+1
  // (element 2k, element 2k+1) times a power of two m, in fp32
  __device__ __forceinline__ float2 scaled(int k, float m) const { return mul_bf16x2_pow2(w[k], m); }
  __device__ __forceinline__ uint32_t signs() const {  // bit i = sign of element i
    uint32_t r = 0;
#pragma unroll
    for (int k = 0; k < 8; k++) r |= ((w[k] >> 15) & 1u) << (2 * k) | (w[k] >> 31) << (2 * k + 1);
    return r;
  }
};

template <>
struct In16<float> {
  uint32_t w[16];
  template <bool V8>
  __device__ __forceinline__ void load(const float* p) {
    if constexpr (V8) {
      uint32_t (&a)[8] = *reinterpret_cast<uint32_t(*)[8]>(&w[0]);
      uint32_t (&b)[8] = *reinterpret_cast<uint32_t(*)[8]>(&w[8]);
      ld_nc_v8(p, a);
      ld_nc_v8(p + 8, b);
    } else {
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const uint4 t = ld_nc_v4(p + 4 * i);
        w[4 * i] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
      }
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 16; i++) w[i] = 0;
  }
  __device__ __forceinline__ float absmax() const {
    float m = fabsf(__uint_as_float(w[0]));
#pragma unroll
    for (int i = 1; i < 16; i++) m = fmaxf(m, fabsf(__uint_as_float(w[i])));
    return m;
  }
  __device__ __forceinline__ float lo(int k) const { return __uint_as_float(w[2 * k]); }
  __device__ __forceinline__ float hi(int k) const { return __uint_as_float(w[2 * k + 1]); }
  __device__ __forceinline__ float2 scaled(int k, float m) const { return mul2(lo(k), hi(k), m); }
  __device__ __forceinline__ uint32_t signs() const {
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) r |= (w[i] >> 31) << i;
    return r;
  }
};

// --------------------------------------------- programmatic dependent launch

// Every kernel starts with this: wait until the grids it depends on (earlier
// work in the stream) have completed and their writes are visible, before any
// global memory access, then allow the next grid in the stream to be
// scheduled. When the kernel was launched without programmatic serialization
// both instructions are no-ops.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches `kernel` with programmatic stream serialization, so its launch and
// CTA scheduling overlap the tail of the previous grid in the stream.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_ex(void (*kernel)(KArgs...), uint32_t grid, uint32_t block,
                                 size_t smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), uint32_t grid, cudaStream_t stream,
                              Args&&... args) {
  return launch_pdl_ex(kernel, grid, kThreads, 0, stream, std::forward<Args>(args)...);
}

// Raises Kernel's dynamic shared memory limit to `bytes` on the current
// device, the first time a call reaches it there (the attribute belongs to the
// device's context, so each device needs its own call).
template <auto Kernel>
inline cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<unsigned char> done[256];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 256 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 256) done[dev].store(1, std::memory_order_release);
  return e;
}

// Multiprocessors of the current device (148 on B200 if the query fails).
inline int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ----------------------------------------------------------- block reduce

// Max over the CTA of a non-negative float (NaN ignored); every thread gets
// the result. `red` is kThreads/32 floats of shared memory.
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; w++) r = fmaxf(r, red[w]);
  return r;
}

}  // namespace mxq
