// common.cuh -- device helpers shared by the epilogue kernels (sm_100a).
//
// Everything on this path is a memory-bound stream: 16-byte vector loads and
// stores that bypass L1 allocation, fp32 arithmetic in registers, and one
// rounding to the storage dtype per output element.  Nothing here is a dense
// contraction, so no tensor-core path exists.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kThreads = 256;  // threads per CTA for every kernel in the library
constexpr int kVec = 8;        // elements per vector unit ("chunk")

// Storage-type tags.  Each knows how to widen 8 consecutive elements to fp32
// and how to round 8 fp32 values (RNE) back.
struct BF16 { using T = uint16_t; static constexpr int kBytes = 2; };
struct F16  { using T = uint16_t; static constexpr int kBytes = 2; };
struct F32  { using T = float;    static constexpr int kBytes = 4; };

// ------------------------------------------------------------ raw access

// 16-byte streaming load through the non-coherent path, no L1 allocation
// (no element is reused), with a 256-byte L2 prefetch hint (a warp reads
// 512 contiguous bytes per load instruction).  MOE_LD_HINT selects other
// cache hints for tuning sweeps.
#ifndef MOE_LD_HINT
#define MOE_LD_HINT 0
#endif
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
#if MOE_LD_HINT == 0
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
#elif MOE_LD_HINT == 1
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
#elif MOE_LD_HINT == 2
  asm("ld.global.nc.L1::no_allocate.L2::128B.v4.u32 {%0,%1,%2,%3}, [%4];"
#else
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
#endif
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// 32-byte form of ld_stream (sm_100 256-bit global access): one instruction
// per lane moves two 16-byte chunks.  The address must be 32-byte aligned.
struct u4x2 { uint4 lo, hi; };
__device__ __forceinline__ u4x2 ld_stream32(const void* p) {
  u4x2 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(v.lo.x), "=r"(v.lo.y), "=r"(v.lo.z), "=r"(v.lo.w),
        "=r"(v.hi.x), "=r"(v.hi.y), "=r"(v.hi.z), "=r"(v.hi.w)
      : "l"(p));
  return v;
}

// 32-byte form of ld_coherent; the address must be 32-byte aligned.
__device__ __forceinline__ u4x2 ld_coherent32(const void* p) {
  u4x2 v;
  asm volatile("ld.global.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v.lo.x), "=r"(v.lo.y), "=r"(v.lo.z), "=r"(v.lo.w),
                 "=r"(v.hi.x), "=r"(v.hi.y), "=r"(v.hi.z), "=r"(v.hi.w)
               : "l"(p)
               : "memory");
  return v;
}

// 16-byte coherent load, no L1 allocation: for data that the same kernel
// also writes (the in-place residual add).
__device__ __forceinline__ uint4 ld_coherent(const void* p) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// 16-byte store, no L1 allocation (MOE_ST_HINT selects other cache hints for
// tuning sweeps).
#ifndef MOE_ST_HINT
#define MOE_ST_HINT 0
#endif
__device__ __forceinline__ void st_stream(void* p, uint4 v) {
#if MOE_ST_HINT == 0
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1,%2,%3,%4};"
#elif MOE_ST_HINT == 1
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
#else
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
#endif
               ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// 32-byte store, no L1 allocation; the address must be 32-byte aligned.
__device__ __forceinline__ void st_stream32(void* p, const uint4& lo, const uint4& hi) {
  asm volatile("st.global.L1::no_allocate.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"l"(p), "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w),
                 "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
               : "memory");
}

// ------------------------------------------------------------ conversions

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2 with round-to-nearest-even; `lo` lands at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

__device__ __forceinline__ uint16_t f32_to_f16(float f) {
  uint16_t r;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// Scalar widen / round for the unaligned (element-granular) paths.
template <class D> __device__ __forceinline__ float load1(const typename D::T* p);
template <> __device__ __forceinline__ float load1<BF16>(const uint16_t* p) {
  return __uint_as_float((uint32_t)__ldg(p) << 16);
}
template <> __device__ __forceinline__ float load1<F16>(const uint16_t* p) {
  return f16_to_f32(__ldg(p));
}
template <> __device__ __forceinline__ float load1<F32>(const float* p) { return __ldg(p); }

// Coherent scalar widen (plain load, for data the kernel may also write).
template <class D> __device__ __forceinline__ float load1c(const typename D::T* p);
template <> __device__ __forceinline__ float load1c<BF16>(const uint16_t* p) {
  return __uint_as_float((uint32_t)*p << 16);
}
template <> __device__ __forceinline__ float load1c<F16>(const uint16_t* p) { return f16_to_f32(*p); }
template <> __device__ __forceinline__ float load1c<F32>(const float* p) { return *p; }

template <class D> __device__ __forceinline__ void store1(typename D::T* p, float v);
template <> __device__ __forceinline__ void store1<BF16>(uint16_t* p, float v) { *p = f32_to_bf16(v); }
template <> __device__ __forceinline__ void store1<F16>(uint16_t* p, float v) { *p = f32_to_f16(v); }
template <> __device__ __forceinline__ void store1<F32>(float* p, float v) { *p = v; }

// Round-trip through the storage dtype (what materialising a tensor does).
template <class D> __device__ __forceinline__ float round_to(float v);
template <> __device__ __forceinline__ float round_to<BF16>(float v) {
  return __uint_as_float((uint32_t)f32_to_bf16(v) << 16);
}
template <> __device__ __forceinline__ float round_to<F16>(float v) {
  return f16_to_f32(f32_to_f16(v));
}
template <> __device__ __forceinline__ float round_to<F32>(float v) { return v; }

// Round two fp32 values to the storage dtype and widen them back, with one
// packed conversion (RNE) for the two.
template <class D> __device__ __forceinline__ void round2(float& a, float& b);
template <> __device__ __forceinline__ void round2<BF16>(float& a, float& b) {
  const uint32_t w = pack_bf16x2(a, b);
  a = bf16_lo(w);
  b = bf16_hi(w);
}
template <> __device__ __forceinline__ void round2<F16>(float& a, float& b) {
  const uint32_t w = pack_f16x2(a, b);
  a = f16_to_f32((uint16_t)(w & 0xffffu));
  b = f16_to_f32((uint16_t)(w >> 16));
}
template <> __device__ __forceinline__ void round2<F32>(float&, float&) {}

// ------------------------------------------------- 8-element vector units

// A chunk of 8 elements in registers as raw bits: one 16-byte word for the
// 16-bit types, two for fp32.
template <class D> struct Raw8 { uint4 w[D::kBytes / 2]; };

// NC = true: read-only streaming path; false: coherent path (data the
// kernel may also write).
template <class D, bool NC = true>
__device__ __forceinline__ Raw8<D> load8(const typename D::T* p) {
  Raw8<D> r;
#pragma unroll
  for (int i = 0; i < D::kBytes / 2; ++i) {
    const uint4* w = reinterpret_cast<const uint4*>(p) + i;
    r.w[i] = NC ? ld_stream(w) : ld_coherent(w);
  }
  return r;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& w, float (&v)[8]) {
  v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
  v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

template <class D> __device__ __forceinline__ void widen8(const Raw8<D>& r, float (&v)[8]);
template <> __device__ __forceinline__ void widen8<BF16>(const Raw8<BF16>& r, float (&v)[8]) {
  unpack_bf16x8(r.w[0], v);
}
template <> __device__ __forceinline__ void widen8<F16>(const Raw8<F16>& r, float (&v)[8]) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(&r.w[0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = f16_to_f32((uint16_t)(u[i] & 0xffffu));
    v[2 * i + 1] = f16_to_f32((uint16_t)(u[i] >> 16));
  }
}
template <> __device__ __forceinline__ void widen8<F32>(const Raw8<F32>& r, float (&v)[8]) {
  v[0] = __uint_as_float(r.w[0].x); v[1] = __uint_as_float(r.w[0].y);
  v[2] = __uint_as_float(r.w[0].z); v[3] = __uint_as_float(r.w[0].w);
  v[4] = __uint_as_float(r.w[1].x); v[5] = __uint_as_float(r.w[1].y);
  v[6] = __uint_as_float(r.w[1].z); v[7] = __uint_as_float(r.w[1].w);
}

// An 8-element chunk with one 32-byte access where A32 and the type is fp32
// (a 32-byte aligned address), else as load8 / store8.
template <class D, bool A32, bool NC = true>
__device__ __forceinline__ Raw8<D> load8a(const typename D::T* p) {
  if constexpr (A32 && D::kBytes == 4) {
    const u4x2 v = NC ? ld_stream32(p) : ld_coherent32(p);
    Raw8<D> r;
    r.w[0] = v.lo;
    r.w[1] = v.hi;
    return r;
  } else {
    return load8<D, NC>(p);
  }
}

// Round 8 fp32 values to a 16-bit storage dtype (RNE), packed into 16 bytes.
template <class D> __device__ __forceinline__ uint4 pack8(const float (&v)[8]);
template <> __device__ __forceinline__ uint4 pack8<BF16>(const float (&v)[8]) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
template <> __device__ __forceinline__ uint4 pack8<F16>(const float (&v)[8]) {
  return make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]),
                    pack_f16x2(v[6], v[7]));
}

// Round 8 fp32 values to the storage dtype (RNE) and store them.
template <class D> __device__ __forceinline__ void store8(typename D::T* p, const float (&v)[8]);
template <> __device__ __forceinline__ void store8<BF16>(uint16_t* p, const float (&v)[8]) {
  st_stream(p, make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                          pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7])));
}
template <> __device__ __forceinline__ void store8<F16>(uint16_t* p, const float (&v)[8]) {
  st_stream(p, make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]),
                          pack_f16x2(v[4], v[5]), pack_f16x2(v[6], v[7])));
}
template <> __device__ __forceinline__ void store8<F32>(float* p, const float (&v)[8]) {
  st_stream(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                          __float_as_uint(v[3])));
  st_stream(p + 4, make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]),
                              __float_as_uint(v[6]), __float_as_uint(v[7])));
}

template <class D, bool A32>
__device__ __forceinline__ void store8a(typename D::T* p, const float (&v)[8]) {
  if constexpr (A32 && D::kBytes == 4) {
    st_stream32(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                              __float_as_uint(v[3])),
                make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                           __float_as_uint(v[7])));
  } else {
    store8<D>(p, v);
  }
}

// ------------------------------------------------------------ math

// Flush-to-zero hardware approximations (one MUFU instruction each):
// ex2.approx.ftz.f32 = 2^x, rcp.approx.ftz.f32 = 1/x, tanh.approx.f32.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_ftz(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;  // log2(e): e^x = 2^(x log2 e)
constexpr float kTwoM32 = 0x1p-32f;

// The logistic function sigma(z) = 1 / (1 + e^-z), evaluated as
//   e  = 2^(-z log2 e)                  (subnormal e, z > 87.3, flushes to 0:
//                                        1 + e rounds to 1 either way)
//   q  = 1 / ((1 + e) * 2^-32)          (scaled so the reciprocal stays a normal
//                                        number for every z > -109, where the
//                                        unscaled one would be subnormal and flush)
//   sigma = q * 2^-32                   (a plain multiply: subnormal sigma kept)
// (1 + e) * 2^-32 is one fused multiply-add, e * 2^-32 + 2^-32, exact up to the
// same single rounding as 1 + e.  For z < -88.7, e = +inf and sigma = 0, as in
// an fp32 evaluation of the definition.  Error: a few fp32 ulp, far below half
// a bf16 ulp.
__device__ __forceinline__ float sigmoid(float z) {
  const float e = ex2_ftz(z * -kLog2e);
  return rcp_ftz(fmaf(e, kTwoM32, kTwoM32)) * kTwoM32;
}

// torch.clamp semantics: a NaN input stays NaN.  PTX min/max with .NaN
// return NaN when an operand is NaN (the limits never are).
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float clamp_max(float v, float hi) { return min_nan(v, hi); }
__device__ __forceinline__ float clamp_sym(float v, float lim) {
  return max_nan(min_nan(v, lim), -lim);
}

// tanh(y) with the hardware approximation (PTX tanh.approx.f32, one MUFU
// instruction).  Its relative error, measured on B200 against float64 over
// [2^-40, 2^4.5) (4096 points per octave), stays below 2^-16.5; the PTX ISA
// bounds it by 2^-10.987.  Either way relu(s tanh(x/s))^2 * p is then within
// a relative 2^-9.98 of the exact value before the final rounding, i.e. within
// one bf16 ulp of the correctly rounded result.
__device__ __forceinline__ float tanh_approx(float y) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(y));
  return t;
}

// Fixed xor-butterfly sum over the 32 lanes of a warp: the same tree every
// call, so the bits do not depend on the grid.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Walks a flat chunk index q over a [rows, cpr] grid in strides of S without
// a division per step: (r, c) = divmod(q, cpr), (dr, dc) = divmod(S, cpr).
struct RowCursor {
  int64_t r, c, dr, dc, cpr;
  __device__ __forceinline__ RowCursor(int64_t q, int64_t stride, int64_t cpr_)
      : r(q / cpr_), c(q % cpr_), dr(stride / cpr_), dc(stride % cpr_), cpr(cpr_) {}
  __device__ __forceinline__ void advance() {
    c += dc;
    r += dr;
    if (c >= cpr) { c -= cpr; r += 1; }
  }
};

// Programmatic dependent launch (PDL).  Every kernel of the library is
// launched with programmatic stream serialisation allowed and begins with
// this prologue: griddepcontrol.wait blocks until the grids this one depends
// on (the previous work in the stream) have completed and their memory is
// visible -- so nothing is read early.  The dependents' trigger is left
// implicit (at CTA exit), so the next kernel's grid is launched as this one
// completes, hiding the launch latency, and its CTAs never share an SM with
// this kernel's running ones.  An explicit launch_dependents at the top
// (MOE_PDL_TRIGGER=1) lets the next grid's CTAs become resident early, where
// a kernel runs fewer CTAs per SM than fit, and wait there: measured on B200
// over the nine-kernel epilogue step, 1154 us per step against 1113 with the
// implicit trigger and 1126 without PDL.  Without a programmatic dependency
// the wait is a no-op.
#ifndef MOE_PDL
#define MOE_PDL 1
#endif
#ifndef MOE_PDL_TRIGGER
#define MOE_PDL_TRIGGER 0
#endif
__device__ __forceinline__ void pdl_prologue() {
#if MOE_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
#if MOE_PDL_TRIGGER
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
#endif
}

// Device-side error word: set bits, never trap.
__device__ __forceinline__ void flag_error(int32_t* err, int32_t bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace moe
