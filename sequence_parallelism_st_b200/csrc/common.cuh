// Shared host/device helpers of libstattn (no kernels).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "stattn.h"

#define ST_API extern "C" __attribute__((visibility("default")))

namespace st {

inline bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Status of the launch just issued on this thread.
inline st_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ST_OK : ST_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is still finishing; it must call
// pdl_wait() before touching global memory that kernel produces or reads.
template <typename... Params, typename... Args>
inline st_status launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return ST_ERR_CUDA;
  }
  return launch_status();
}

// Device side of the dependent launch: let the next kernel of the stream be
// scheduled, and wait until the previous one has finished (its writes are
// visible).  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// A pointer the compiler cannot see through: loads through the result depend
// on this point of the program.  Every input read after pdl_wait() goes
// through it, since loads through const __restrict__ pointers (and __ldg) are
// taken as invariant and could otherwise be scheduled before the wait.
template <typename T>
__device__ __forceinline__ T *after_wait(T *p) {
  asm volatile("" : "+l"(p));
  return p;
}

// SM count of the current device (cached per device ordinal).
int num_sms();

// Reads and clears the device error word of the tensor-core attention kernel
// (defined next to that kernel).  Returns the word's previous value.
unsigned int read_and_clear_attn_error(cudaStream_t stream, cudaError_t *err);
unsigned int read_and_clear_relayout_error(cudaStream_t stream, cudaError_t *err);
unsigned int read_and_clear_vmajor_error(cudaStream_t stream, cudaError_t *err);

// Division of 0 <= n < 2^31 by a divisor fixed for the launch, as a multiply
// and a shift: with l = ceil(log2 d) and m = ceil(2^(31+l) / d) (< 2^32),
// floor(n / d) = (n * m) >> (31 + l) exactly (Granlund and Montgomery,
// "Division by invariant integers using multiplication", theorem 4.2: the
// error m d - 2^(31+l) is below 2^l).  Integer division by a runtime value
// would otherwise take a reciprocal on the special-function pipe and about a
// dozen more instructions.
struct FastDiv {
  uint32_t d, m, shift;
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  const unsigned long long num = 1ull << (31 + l);
  return FastDiv{d, uint32_t((num + d - 1) / d), 31 + l};
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
  return uint32_t((unsigned long long)n * f.m >> f.shift);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// Round to nearest even; NaN stays NaN.
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// The (cos, sin) pairs of one 16-byte vector of a head (EPV / 2 pairs, 16-byte
// aligned in the table): two 16-byte reads for bf16, one for fp32.
template <typename T> struct RotVec {
  float4 c[sizeof(T) == 2 ? 2 : 1];
};
template <typename T> __device__ __forceinline__ RotVec<T> load_rot(const float2 *rot) {
  RotVec<T> r;
#pragma unroll
  for (int i = 0; i < (sizeof(T) == 2 ? 2 : 1); ++i) r.c[i] = reinterpret_cast<const float4 *>(rot)[i];
  return r;
}

// One 16-byte vector of a head on its way through the per-head RMSNorm and,
// with ROPE, the rotary position embedding: every element x becomes
// y = x * inv * g, then pair k of the vector (elements 2k, 2k+1, pair index
// u * EPV / 2 + k of the head) turns by the angle whose (cos, sin) is pair k
// of cs:  (y0, y1) -> (y0 c - y1 s, y0 s + y1 c).  T: uint16_t (bf16) or
// float.  The rotation is a compile-time choice, so a kernel without it holds
// no table load at all; kernels load cs (load_rot) a few vectors ahead.
template <typename T, bool ROPE>
__device__ __forceinline__ uint4 rms_rope_vec(uint4 v, float inv, const float *gg, const RotVec<T> &cs) {
  if constexpr (sizeof(T) == 2) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a = __uint_as_float(w[k] << 16) * inv * gg[2 * k];
      float b = __uint_as_float(w[k] & 0xffff0000u) * inv * gg[2 * k + 1];
      if constexpr (ROPE) {
        const float4 c = cs.c[k >> 1];
        const float2 r = (k & 1) ? make_float2(c.z, c.w) : make_float2(c.x, c.y);
        const float a2 = a * r.x - b * r.y;
        b = a * r.y + b * r.x;
        a = a2;
      }
      w[k] = pack_bf16x2(a, b);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    float y[4] = {__uint_as_float(v.x) * inv * gg[0], __uint_as_float(v.y) * inv * gg[1],
                  __uint_as_float(v.z) * inv * gg[2], __uint_as_float(v.w) * inv * gg[3]};
    if constexpr (ROPE) {
      const float4 c = cs.c[0];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float2 r = k ? make_float2(c.z, c.w) : make_float2(c.x, c.y);
        const float a = y[2 * k], b = y[2 * k + 1];
        y[2 * k] = a * r.x - b * r.y;
        y[2 * k + 1] = a * r.y + b * r.x;
      }
    }
    return make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]), __float_as_uint(y[3]));
  }
}

// Rotation table reads of a head, RG vectors at a time: the normalise loop of
// the RMSNorm kernels loads the pairs of RG vectors together (one round trip
// per group instead of one per vector), the first group before the head's sum
// of squares.
constexpr int RG = 4;

}  // namespace st
