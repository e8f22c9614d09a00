// FP8 (e4m3) quantisation of bf16 rows with one power-of-two scale per group of rows, for the
// FP8 logit product of the attention.
//
// Spark-H3 blog, section "Benchmark Results": Spark-H3's attention is also timed in FP8; the
// scheme is not described.  Reading taken here: the queries, the exact keys, the summary keys
// and the context keys enter the logit product as e4m3 (OCP E4M3FN: bias 7, 3 mantissa
// bits, largest finite 448), one scale 2^e per group of rows - a query block, a key block, or
// a 128-row tile of summary or context rows - with e the smallest integer such that the
// group's largest |value| is at most 448 * 2^e (at least -126; 0 for an all-zero group).
// x * 2^-e is then exact in fp32 and is rounded to e4m3 to nearest, ties to even, saturating.
//
// One CTA per (group, head), 256 threads; rows of d bf16 are read as 16-byte chunks of 8
// values, twice (maximum, then codes; the second read hits L2), and written as 8-byte chunks
// of 8 codes.
#include <cuda_fp8.h>

#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kQuantThreads = 256;

// The smallest e >= -126 with amax <= 448 * 2^e (0 when amax is 0 or not finite).
// amax = m * 2^x with m in [0.5, 1) and 448 = 0.875 * 2^9: the bound holds for e = x - 9 when
// m <= 0.875, else first for e = x - 8.
__device__ __forceinline__ int group_exponent(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 0;
  int x;
  const float m = frexpf(amax, &x);
  const int e = (m <= 0.875f) ? x - 9 : x - 8;
  return max(e, -126);
}

__global__ void __launch_bounds__(kQuantThreads) quant_fp8_kernel(
    const __nv_bfloat16* __restrict__ src, int R, int d, const int32_t* __restrict__ offsets,
    int ngroups, uint8_t* __restrict__ dst, float* __restrict__ scales, uint32_t* err) {
  __shared__ float s_max[kQuantThreads / 32];
  const int g = blockIdx.x, h = blockIdx.y;
  int lo, hi;
  if (offsets != nullptr) {
    lo = offsets[g];
    hi = offsets[g + 1];
    if (lo < 0 || hi > R || hi < lo) {           // bad offsets: nothing is read or written
      if (threadIdx.x == 0) {
        flag_error(err, kErrOffsets);
        scales[static_cast<size_t>(h) * ngroups + g] = 1.f;
      }
      return;
    }
  } else {
    lo = g * 128;
    hi = min(lo + 128, R);
  }
  const int cpr = d / 8;                          // 16-byte chunks per row
  const int nchunks = (hi - lo) * cpr;
  const size_t base = (static_cast<size_t>(h) * R + lo) * d;
  const uint4* in = reinterpret_cast<const uint4*>(src + base);
  float amax = 0.f;
  for (int i = threadIdx.x; i < nchunks; i += kQuantThreads) {
    const uint4 v = in[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = s_max[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, s_max[w]);
  const int e = group_exponent(amax);
  const float inv = ldexpf(1.f, -e);              // exact power of two
  if (threadIdx.x == 0) scales[static_cast<size_t>(h) * ngroups + g] = ldexpf(1.f, e);
  uint2* out = reinterpret_cast<uint2*>(dst + base);
  for (int i = threadIdx.x; i < nchunks; i += kQuantThreads) {
    const uint4 v = in[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(w[j] << 16) * inv;          // element 2j
      const float b = __uint_as_float(w[j] & 0xFFFF0000u) * inv;  // element 2j+1
      const uint32_t ca = __nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
      const uint32_t cb = __nv_cvt_float_to_fp8(b, __NV_SATFINITE, __NV_E4M3);
      packed[j >> 1] |= (ca | (cb << 8)) << ((j & 1) * 16);
    }
    out[i] = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace

cudaError_t launch_quant_fp8(const void* src, int H, int R, int d, const int32_t* offsets,
                             int ngroups, void* dst, float* scales, uint32_t* err,
                             cudaStream_t s) {
  if (ngroups <= 0 || R <= 0) return cudaSuccess;
  dim3 grid(ngroups, H);
  quant_fp8_kernel<<<grid, kQuantThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(src), R, d,
                                                  offsets, ngroups,
                                                  static_cast<uint8_t*>(dst), scales, err);
  return cudaGetLastError();
}

}  // namespace spark
