// Device-side helpers shared by the cplse kernels: 16-byte payload vectors,
// bf16/fp16 <-> fp32 conversion, read-only loads, streaming stores.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cplse {

constexpr int kVecBytes = 16;   // one load/store: 8 payload elements
constexpr int kVecElems = 8;

struct Bf16 {};
struct Fp16 {};

// Two payload elements packed in one 32-bit word (element 2k in the low half).
template <typename P>
__device__ __forceinline__ float2 unpack2(uint32_t w);

template <>
__device__ __forceinline__ float2 unpack2<Bf16>(uint32_t w)
{
    // bf16 is the upper half of an fp32: shifting is an exact conversion.
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <>
__device__ __forceinline__ float2 unpack2<Fp16>(uint32_t w)
{
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
}

// Round two fp32 to the payload format, nearest-even.
template <typename P>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);

template <>
__device__ __forceinline__ uint32_t pack2<Bf16>(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <>
__device__ __forceinline__ uint32_t pack2<Fp16>(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Loads of inputs that nothing writes while the kernel runs: the read-only
// (non-coherent) path with the default cache policy. The merge kernels read
// every input byte exactly once, yet the evict-first hint (ld.global.cs) made
// them slower: on a 16-rank fp16 merge 2966 against 2861 us, on its combine
// 2888 against 2735 us, and an 8-rank bf16 merge ran either at 1400 or at
// 1505 us depending on what had run on the GPU before it; with this path it
// runs at 1400 us from the first call. Same bits either way.
__device__ __forceinline__ uint4 ld_ro(const uint4* p) { return __ldg(p); }
__device__ __forceinline__ float ld_ro(const float* p) { return __ldg(p); }
__device__ __forceinline__ void st_stream(uint4* p, uint4 v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(float* p, float v) { __stcs(p, v); }

}  // namespace cplse
