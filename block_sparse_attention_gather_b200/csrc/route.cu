// Block scoring + per-query-block Top-K (Spark-H3 blog, "Discussion": blocks are scored from
// block-level means; "Spark-Reblock": a fixed Top-K budget of key blocks per query block).
//
// One CTA per (R consecutive query blocks, head), 512 threads:
//   phase 1  S[r, B] = qbar_A(r) . kbar_B in fp32 (sequential FMA over d) for every key
//            block.  A thread owns two key blocks at a time: their means stream through its
//            registers in 8-dimension chunks straight from global memory (L2-resident: every
//            CTA of the head reads them; kbar is stored d-major, so a warp's load is one
//            coalesced row of 32 key blocks), the next chunk in flight while the current one
//            is used, and the R query rows come from shared memory stored d-major, so each
//            load is a warp-wide broadcast of four rows.  The scores of the R
//            rows stay in shared memory as order-preserving uint32 keys.  The positive factor
//            1/sqrt(d) is left out: it does not change the order.
//   phase 2  one warp per row: an exact radix select (four 8-bit passes over the keys) finds
//            the k-th largest key T and how many keys equal to T are still needed; a ballot
//            scan in ascending block order then writes every B with key > T and the
//            lowest-indexed keys == T, so the selection is stored ascending and ties go to
//            the smaller block index.
#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kCols = 2;          // key blocks a thread scores at once
constexpr int kChunk = 16;        // d-elements of each kbar_B held in registers at a time
constexpr bool kPrefetch = true;  // load the next chunk while the current one is in use

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ float4 ld_nc_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

}  // namespace

// kThreshold: Sol-Attn-style routing (the blog's "Discussion": block logits taken as roughly
// Gaussian, the blocks above mu + tau*sigma exact) instead of the fixed Top-K budget.  Per row:
// mu and the population sigma of the row's nkb scores (two passes, fp32; the positive factor
// 1/sqrt(d) left out of the scores moves mu + tau*sigma with them), the count of scores strictly
// above the threshold, capped at k (the largest kept, ties to the smaller block, as Top-K); the
// selection is written to the first count entries of the row (rows are k apart) and the count
// to count[h, A].
template <int D, int R, bool kThreshold>
__global__ void __launch_bounds__(kThreads, 1) route_kernel(const float* __restrict__ qbar_blocks,
                                                            const float* __restrict__ kbar,
                                                            int nqb, int nkb, int k, float tau,
                                                            int32_t* __restrict__ sel,
                                                            int32_t* __restrict__ count) {
  static_assert(R % 4 == 0 && D % kChunk == 0, "tile shape");
  extern __shared__ __align__(16) float sm[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm);     // [R][nkb]
  float* qT = sm + static_cast<size_t>(R) * nkb;        // [D][R]  (R*nkb*4 is 16-byte aligned)
  uint32_t* hist = reinterpret_cast<uint32_t*>(qT + D * R);  // [kWarps][256]

  const int h = blockIdx.y;
  const int A0 = blockIdx.x * R;
  const int rows = min(R, nqb - A0);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  for (int i = tid; i < R * D; i += kThreads) {
    const int r = i / D, e = i % D;
    qT[e * R + r] = (r < rows) ? qbar_blocks[(static_cast<size_t>(h) * nqb + A0 + r) * D + e] : 0.f;
  }
  __syncthreads();

  // ---- phase 1: scores (no collectives inside: the ragged last pass needs no uniformity)
  // kbar is d-major ([D][nkb] per head): the threads of a warp read consecutive key blocks of
  // one dimension, one coalesced 128-byte row per load.
  const float* kbT = kbar + static_cast<size_t>(h) * D * nkb;
  for (int B0 = tid; B0 < nkb; B0 += kCols * kThreads) {
    float acc[kCols][R];
    int Bc[kCols];
    bool live[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      live[c] = B0 + c * kThreads < nkb;
      Bc[c] = live[c] ? B0 + c * kThreads : B0;
#pragma unroll
      for (int r = 0; r < R; ++r) acc[c][r] = 0.f;
    }
    float b[kCols][kChunk];
#pragma unroll
    for (int c = 0; c < kCols; ++c)
#pragma unroll
      for (int j = 0; j < kChunk; ++j) b[c][j] = __ldg(kbT + static_cast<size_t>(j) * nkb + Bc[c]);
#pragma unroll 1
    for (int e0 = 0; e0 < D; e0 += kChunk) {
      float nb[kCols][kChunk];
      if (kPrefetch && e0 + kChunk < D) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            nb[c][j] = __ldg(kbT + static_cast<size_t>(e0 + kChunk + j) * nkb + Bc[c]);
      }
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        const float4* a = reinterpret_cast<const float4*>(qT + (e0 + j) * R);
#pragma unroll
        for (int r4 = 0; r4 < R / 4; ++r4) {
          const float4 av = a[r4];
#pragma unroll
          for (int c = 0; c < kCols; ++c) {
            const float bv = b[c][j];
            acc[c][4 * r4 + 0] = fmaf(av.x, bv, acc[c][4 * r4 + 0]);
            acc[c][4 * r4 + 1] = fmaf(av.y, bv, acc[c][4 * r4 + 1]);
            acc[c][4 * r4 + 2] = fmaf(av.z, bv, acc[c][4 * r4 + 2]);
            acc[c][4 * r4 + 3] = fmaf(av.w, bv, acc[c][4 * r4 + 3]);
          }
        }
      }
      if (e0 + kChunk < D) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            b[c][j] = kPrefetch ? nb[c][j]
                                : __ldg(kbT + static_cast<size_t>(e0 + kChunk + j) * nkb + Bc[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < kCols; ++c)
      if (live[c]) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          keys[static_cast<size_t>(r) * nkb + B0 + c * kThreads] = order_key(acc[c][r]);
      }
  }
  __syncthreads();

  // ---- phase 2: exact Top-K per row, one warp per row
  uint32_t* wh = hist + warp * 256;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; r < rows; r += kWarps) {
    const uint32_t* krow = keys + static_cast<size_t>(r) * nkb;
    int32_t* out = sel + (static_cast<size_t>(h) * nqb + A0 + r) * k;
    int kr = k;                        // blocks this row takes
    if constexpr (kThreshold) {
      float sum = 0.f;
      for (int B = lane; B < nkb; B += 32) sum += key_value(krow[B]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const float mu = sum / static_cast<float>(nkb);
      float ss = 0.f;
      for (int B = lane; B < nkb; B += 32) {
        const float dv = key_value(krow[B]) - mu;
        ss = fmaf(dv, dv, ss);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float thr = fmaf(tau, sqrtf(ss / static_cast<float>(nkb)), mu);
      const uint32_t tkey = order_key(thr);
      int above = 0;
      for (int B0 = 0; B0 < nkb; B0 += 32) {
        const int B = B0 + lane;
        above += __popc(__ballot_sync(0xffffffffu, B < nkb && krow[min(B, nkb - 1)] > tkey));
      }
      kr = min(above, k);
      if (lane == 0) count[static_cast<size_t>(h) * nqb + A0 + r] = kr;
      if (kr == 0) continue;           // uniform: nothing to write
    }
    uint32_t prefix = 0, pmask = 0;
    int need = kr;                     // still to take among keys matching `prefix`
    if (kr < nkb) {
      // digits shared by every key of the row (a row's scores share their top bits) are known
      // without a histogram: start at the first digit where the smallest and largest key differ
      uint32_t kmin = 0xffffffffu, kmax = 0u;
      for (int B = lane; B < nkb; B += 32) {
        const uint32_t u = krow[B];
        kmin = min(kmin, u);
        kmax = max(kmax, u);
      }
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      int shift0 = 24;
      while (shift0 > 0 && ((kmin ^ kmax) >> shift0) == 0u) {
        prefix |= kmin & (255u << shift0);
        pmask |= 255u << shift0;
        shift0 -= 8;
      }
      for (int shift = shift0; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) wh[i] = 0;
        __syncwarp();
        for (int B = lane; B < nkb; B += 32) {
          const uint32_t u = krow[B];
          if ((u & pmask) == prefix) atomicAdd(&wh[(u >> shift) & 255u], 1u);
        }
        __syncwarp();
        // lane l owns digits [8l, 8l+8); suffix sums give count(digit >= x)
        uint32_t c[8], local = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = wh[lane * 8 + j];
          local += c[j];
        }
        uint32_t suf = local;          // inclusive suffix scan over lanes
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t v = __shfl_down_sync(0xffffffffu, suf, off);
          if (lane + off < 32) suf += v;
        }
        uint32_t above = suf - local;  // count(digit >= 8(l+1))
        int best = -1;
        uint32_t best_gt = 0;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          const uint32_t ge = above + c[j];
          if (best < 0 && ge >= static_cast<uint32_t>(need)) {
            best = lane * 8 + j;
            best_gt = above;
          }
          above = ge;
        }
        // the selected digit is the largest x with count(>= x) >= need
        const int dd = __reduce_max_sync(0xffffffffu, best);
        const uint32_t gt = __shfl_sync(0xffffffffu, best_gt, dd / 8);
        need -= static_cast<int>(gt);
        prefix |= static_cast<uint32_t>(dd) << shift;
        pmask |= 255u << shift;
        const bool all_taken = static_cast<uint32_t>(need) == wh[dd];
        __syncwarp();
        // every key left under the prefix is taken: the remaining digits cannot change the set
        if (all_taken) break;
      }
    } else {
      prefix = 0;                      // k == nkb: every key is taken
      need = nkb;
    }
    const uint32_t T = prefix;         // compared on the resolved digits only
    int taken = 0, eq_seen = 0;
    for (int B0 = 0; B0 < nkb; B0 += 32) {
      const int B = B0 + lane;
      const uint32_t u = ((B < nkb) ? krow[B] : 0u) & pmask;
      const bool valid = B < nkb;
      const bool gt = valid && (kr == nkb || u > T);
      const bool eq = valid && kr < nkb && u == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqb & lt_mask);
      const bool take = gt || (eq && eq_rank < need);
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      if (take) out[taken + __popc(tb & lt_mask)] = B;
      taken += __popc(tb);
      eq_seen += __popc(eqb);
    }
  }
}

template <int D, int R>
constexpr size_t route_smem_bytes(int nkb) {
  return (static_cast<size_t>(R) * nkb + R * D) * 4 + kWarps * 256 * 4;
}

constexpr size_t kRouteSmemLimit = 232448;   // 227 KB of opt-in shared memory per CTA

template <int D, int R, bool kThreshold>
static cudaError_t launch_route_t(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                  int nkb, int k, float tau, int32_t* sel, int32_t* count,
                                  cudaStream_t s) {
  const size_t smem = route_smem_bytes<D, R>(nkb);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<D, R, kThreshold>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((nqb + R - 1) / R, H);
  route_kernel<D, R, kThreshold><<<grid, kThreads, smem, s>>>(qbar_blocks, kbar, nqb, nkb, k,
                                                              tau, sel, count);
  return cudaGetLastError();
}

template <int D, bool kThreshold>
static cudaError_t launch_route_d(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                  int nkb, int k, float tau, int32_t* sel, int32_t* count,
                                  cudaStream_t s) {
  if (route_smem_bytes<D, 16>(nkb) <= kRouteSmemLimit)
    return launch_route_t<D, 16, kThreshold>(qbar_blocks, kbar, H, nqb, nkb, k, tau, sel, count,
                                             s);
  if (route_smem_bytes<D, 8>(nkb) <= kRouteSmemLimit)
    return launch_route_t<D, 8, kThreshold>(qbar_blocks, kbar, H, nqb, nkb, k, tau, sel, count,
                                            s);
  return launch_route_t<D, 4, kThreshold>(qbar_blocks, kbar, H, nqb, nkb, k, tau, sel, count, s);
}

cudaError_t launch_route(const float* qbar_blocks, const float* kbar, int H, int nqb, int nkb,
                         int d, int k, int32_t* sel, uint32_t* /*err*/, cudaStream_t s) {
  if (d == 128)
    return launch_route_d<128, false>(qbar_blocks, kbar, H, nqb, nkb, k, 0.f, sel, nullptr, s);
  return launch_route_d<64, false>(qbar_blocks, kbar, H, nqb, nkb, k, 0.f, sel, nullptr, s);
}

cudaError_t launch_route_threshold(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                   int nkb, int d, float tau, int kcap, int32_t* sel,
                                   int32_t* count, cudaStream_t s) {
  if (d == 128)
    return launch_route_d<128, true>(qbar_blocks, kbar, H, nqb, nkb, kcap, tau, sel, count, s);
  return launch_route_d<64, true>(qbar_blocks, kbar, H, nqb, nkb, kcap, tau, sel, count, s);
}

}  // namespace spark
