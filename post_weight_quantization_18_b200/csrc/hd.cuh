// hd.cuh — macros of the host-and-device helper headers (pack32.cuh, gather4.cuh,
// tri_fill.cuh), which compile both into the kernels and into the CPU checks under tests/c.
#pragma once

#if defined(__CUDACC__)
#define GPTQ_HD __host__ __device__ __forceinline__
#else
#define GPTQ_HD inline
#endif

#if defined(__CUDA_ARCH__)
#define GPTQ_UNROLL _Pragma("unroll")
#else
#define GPTQ_UNROLL
#endif
