// Block scoring + per-query-block Top-K (Spark-H3 blog, "Discussion": blocks are scored from
// block-level means; "Spark-Reblock": a fixed Top-K budget of key blocks per query block).
//
// One CTA per (R consecutive query blocks, head), 256 threads:
//   phase 1  S[r, B] = qbar_A(r) . kbar_B in fp32 (sequential FMA over d) for every key
//            block, staged through shared memory in 32-block tiles; the scores of the R
//            rows stay in shared memory.  The positive factor 1/sqrt(d) is left out: it does
//            not change the order.
//   phase 2  one warp per row: an exact radix select (four 8-bit passes over the
//            order-preserving uint32 image of the fp32 score) finds the k-th largest key T
//            and how many keys equal to T are still needed; a ballot scan in ascending block
//            order then writes every B with key > T and the lowest-indexed keys == T, so the
//            selection is stored ascending and ties go to the smaller block index.
#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kThreads = 256;
constexpr int kTileCols = 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace

template <int D, int R>
__global__ void __launch_bounds__(kThreads) route_kernel(const float* __restrict__ qbar_blocks,
                                                         const float* __restrict__ kbar, int nqb,
                                                         int nkb, int k,
                                                         int32_t* __restrict__ sel) {
  extern __shared__ __align__(16) float sm[];
  float* scores = sm;                                   // [R][nkb]
  float* qrows = scores + static_cast<size_t>(R) * nkb; // [R][D]
  float* ktile = qrows + R * D;                         // [kTileCols][D + 1]
  uint32_t* hist = reinterpret_cast<uint32_t*>(ktile + kTileCols * (D + 1));  // [8][256]

  const int h = blockIdx.y;
  const int A0 = blockIdx.x * R;
  const int rows = min(R, nqb - A0);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  for (int i = tid; i < R * D; i += kThreads) {
    const int r = i / D;
    qrows[i] = (r < rows) ? qbar_blocks[(static_cast<size_t>(h) * nqb + A0 + r) * D + i % D] : 0.f;
  }

  // ---- phase 1: scores
  constexpr int OUT_PER_THREAD = (R * kTileCols) / kThreads;   // 2 (R=16), 1 (R=8)
  constexpr int RSTEP = kThreads / kTileCols;                  // 8 rows per pass
  const float* kb = kbar + static_cast<size_t>(h) * nkb * D;
  for (int B0 = 0; B0 < nkb; B0 += kTileCols) {
    __syncthreads();
    for (int i = tid; i < kTileCols * D; i += kThreads) {
      const int cb = i / D, e = i % D;
      ktile[cb * (D + 1) + e] = (B0 + cb < nkb) ? kb[static_cast<size_t>(B0 + cb) * D + e] : 0.f;
    }
    __syncthreads();
    const int col = tid % kTileCols;
    const int r0 = tid / kTileCols;
    if (B0 + col < nkb) {
      if constexpr (OUT_PER_THREAD >= 1) {
        float acc[OUT_PER_THREAD > 0 ? OUT_PER_THREAD : 1];
#pragma unroll
        for (int o = 0; o < OUT_PER_THREAD; ++o) acc[o] = 0.f;
        const float* kr = ktile + col * (D + 1);
#pragma unroll 8
        for (int e = 0; e < D; ++e) {
          const float kv = kr[e];
#pragma unroll
          for (int o = 0; o < OUT_PER_THREAD; ++o) acc[o] = fmaf(qrows[(r0 + o * RSTEP) * D + e], kv, acc[o]);
        }
#pragma unroll
        for (int o = 0; o < OUT_PER_THREAD; ++o)
          scores[static_cast<size_t>(r0 + o * RSTEP) * nkb + B0 + col] = acc[o];
      } else {
        if (r0 < R) {
          float acc = 0.f;
          const float* kr = ktile + col * (D + 1);
#pragma unroll 8
          for (int e = 0; e < D; ++e) acc = fmaf(qrows[r0 * D + e], kr[e], acc);
          scores[static_cast<size_t>(r0) * nkb + B0 + col] = acc;
        }
      }
    }
  }
  __syncthreads();

  // ---- phase 2: exact Top-K per row, one warp per row
  uint32_t* wh = hist + warp * 256;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; r < rows; r += kThreads / 32) {
    const float* srow = scores + static_cast<size_t>(r) * nkb;
    int32_t* out = sel + (static_cast<size_t>(h) * nqb + A0 + r) * k;
    uint32_t prefix = 0, pmask = 0;
    int need = k;                      // still to take among keys matching `prefix`
    if (k < nkb) {
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) wh[i] = 0;
        __syncwarp();
        for (int B = lane; B < nkb; B += 32) {
          const uint32_t u = order_key(srow[B]);
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
        __syncwarp();
      }
    } else {
      prefix = 0;                      // k == nkb: every key is taken
      need = nkb;
    }
    const uint32_t T = prefix;
    int taken = 0, eq_seen = 0;
    for (int B0 = 0; B0 < nkb; B0 += 32) {
      const int B = B0 + lane;
      const uint32_t u = (B < nkb) ? order_key(srow[B]) : 0u;
      const bool valid = B < nkb;
      const bool gt = valid && (k == nkb || u > T);
      const bool eq = valid && k < nkb && u == T;
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
  return (static_cast<size_t>(R) * nkb + R * D + kTileCols * (D + 1)) * 4 + 8 * 256 * 4;
}

constexpr size_t kRouteSmemLimit = 232448;   // 227 KB of opt-in shared memory per CTA

template <int D, int R>
static cudaError_t launch_route_t(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                  int nkb, int k, int32_t* sel, cudaStream_t s) {
  const size_t smem = route_smem_bytes<D, R>(nkb);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<D, R>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((nqb + R - 1) / R, H);
  route_kernel<D, R><<<grid, kThreads, smem, s>>>(qbar_blocks, kbar, nqb, nkb, k, sel);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_route_d(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                  int nkb, int k, int32_t* sel, cudaStream_t s) {
  if (route_smem_bytes<D, 16>(nkb) <= kRouteSmemLimit)
    return launch_route_t<D, 16>(qbar_blocks, kbar, H, nqb, nkb, k, sel, s);
  if (route_smem_bytes<D, 8>(nkb) <= kRouteSmemLimit)
    return launch_route_t<D, 8>(qbar_blocks, kbar, H, nqb, nkb, k, sel, s);
  return launch_route_t<D, 4>(qbar_blocks, kbar, H, nqb, nkb, k, sel, s);
}

cudaError_t launch_route(const float* qbar_blocks, const float* kbar, int H, int nqb, int nkb,
                         int d, int k, int32_t* sel, uint32_t* /*err*/, cudaStream_t s) {
  if (d == 128) return launch_route_d<128>(qbar_blocks, kbar, H, nqb, nkb, k, sel, s);
  return launch_route_d<64>(qbar_blocks, kbar, H, nqb, nkb, k, sel, s);
}

}  // namespace spark
