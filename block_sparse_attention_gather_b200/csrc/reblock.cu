// Spark-Reblock token partitioner (Spark-H3 blog, section "Spark-Reblock").
//
// Queries are grouped under the Mahalanobis cosine distance d_Q(q_i, q_j) =
// 1 - cos(M_K^{1/2} q_i, M_K^{1/2} q_j), M_K = E[k k^T] (keys symmetrically, with M_Q).  A
// hierarchical partitioner splits every group level by level into children of assigned
// capacities until every leaf is one block.  The split rule is not spelled out in the blog;
// this implementation takes the following reading:
//   - fixed-size blocks (the last takes the remainder); a binary tree over the block range
//     whose nodes give ceil(m/2) blocks to the left child;
//   - a node splits along the principal direction of its unit vectors x_i = W q_i / |W q_i|
//     (W = M^{1/2}), estimated by kPowerIters power iterations of the node covariance from
//     v0 = (1,...,1)/sqrt(d); the left child takes its capacity of largest projections,
//     equal projections go to the token earlier in the node's current order, and both
//     children keep the current relative order.
//
// Steps and kernels (one stream):
//   prepare   rb_moment_partial + rb_moment_reduce   M = (1/N) sum_j y_j y_j^T (fixed order)
//             rb_sqrt                                W = M^{1/2}: coupled Newton-Schulz
//                                                    iteration, one CTA per head, in smem
//             rb_whiten                              X = rows W x_i / |W x_i| (bf16)
//   per level (all heads and all nodes of the level at once; nodes cut into chunks of
//             kChunk tokens so that big nodes spread over many CTAs):
//             rb_power + rb_node_reduce (x kPowerIters)  fixed-order partial sums
//             rb_project, then rb_pick / rb_hist       exact radix select (4 x 8 bits) of
//                                                      the capacity-th largest projection
//             rb_count, rb_scan, rb_scatter            stable two-way partition of perm
// Everything is deterministic: sums run in a fixed order, histograms are integer counts.
#include <cmath>
#include <type_traits>
#include <vector>

#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kRbThreads = 256;
constexpr int kRbWarps = kRbThreads / 32;
constexpr int kChunk = 1024;        // tokens of one node handled by one CTA
constexpr int kPowerIters = 4;
constexpr int kNsIters = 40;        // Newton-Schulz iterations at most
constexpr float kNsTol = 1e-5f;     // stop once max |Z Y - I| is below this
constexpr int kMomentParts = 16;    // row partitions of the second-moment sum per head
constexpr int kRowsInFlight = 8;    // unit rows a warp loads before using them

__device__ __forceinline__ uint32_t rb_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace

// ------------------------------------------------------------------ second moment
// part[h][p] = sum over rows [N p / P, N (p+1) / P) of y y^T; thread (ib, jb) owns the
// TI x TI tile of rows ib*TI.., columns jb*TI.. and accumulates rows in order.
template <int D, typename T>
__global__ void __launch_bounds__(kRbThreads) rb_moment_partial_kernel(const T* __restrict__ Y,
                                                                       int N,
                                                                       float* __restrict__ part) {
  constexpr int TI = D / 16;
  constexpr int ROWS = 32;
  __shared__ __align__(16) float tile[ROWS][D];
  const int h = blockIdx.y, p = blockIdx.x, P = gridDim.x;
  const int r0 = static_cast<int>(static_cast<long long>(N) * p / P);
  const int r1 = static_cast<int>(static_cast<long long>(N) * (p + 1) / P);
  const int ib = threadIdx.x / 16, jb = threadIdx.x % 16;
  float acc[TI][TI];
#pragma unroll
  for (int i = 0; i < TI; ++i)
#pragma unroll
    for (int j = 0; j < TI; ++j) acc[i][j] = 0.f;
  const T* Yh = Y + static_cast<size_t>(h) * N * D;
  for (int base = r0; base < r1; base += ROWS) {
    const int nr = min(ROWS, r1 - base);
    __syncthreads();
    for (int i = threadIdx.x; i < ROWS * D; i += kRbThreads) {
      const int r = i / D, e = i % D;
      tile[r][e] = r < nr ? ld_f(Yh + static_cast<size_t>(base + r) * D + e) : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      float a[TI], b[TI];
#pragma unroll
      for (int t = 0; t < TI; t += 4) {
        const float4 av = *reinterpret_cast<const float4*>(&tile[r][ib * TI + t]);
        const float4 bv = *reinterpret_cast<const float4*>(&tile[r][jb * TI + t]);
        a[t] = av.x; a[t + 1] = av.y; a[t + 2] = av.z; a[t + 3] = av.w;
        b[t] = bv.x; b[t + 1] = bv.y; b[t + 2] = bv.z; b[t + 3] = bv.w;
      }
#pragma unroll
      for (int i = 0; i < TI; ++i)
#pragma unroll
        for (int j = 0; j < TI; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
  float* out = part + (static_cast<size_t>(h) * P + p) * D * D;
#pragma unroll
  for (int i = 0; i < TI; ++i)
#pragma unroll
    for (int j = 0; j < TI; ++j) out[(ib * TI + i) * D + jb * TI + j] = acc[i][j];
}

template <int D>
__global__ void __launch_bounds__(kRbThreads) rb_moment_reduce_kernel(const float* __restrict__ part,
                                                                      int P, int N,
                                                                      float* __restrict__ M) {
  const int h = blockIdx.x;
  const float inv = 1.f / static_cast<float>(N);
  for (int idx = threadIdx.x; idx < D * D; idx += kRbThreads) {
    float s = 0.f;
    for (int p = 0; p < P; ++p) s += part[(static_cast<size_t>(h) * P + p) * D * D + idx];
    M[static_cast<size_t>(h) * D * D + idx] = s * inv;
  }
}

// ------------------------------------------------------------------ W = M^{1/2}
// Coupled Newton-Schulz iteration (stable form): with c = |M|_F (>= the largest eigenvalue
// of a PSD M), Y0 = M/c, Z0 = I, T = (3I - Z Y)/2, Y <- Y T, Z <- T Z; Y converges to
// (M/c)^{1/2} and W = sqrt(c) Y.  Zero eigenvalues stay zero.  The loop stops once
// max |Z Y - I| < kNsTol (a block-wide decision, so the count depends only on M) or after
// kNsIters steps.  One CTA per head, the three D x D matrices in shared memory; thread
// (rg, cg) owns a RT x CT tile of every product.
template <int D>
__global__ void __launch_bounds__(512) rb_sqrt_kernel(const float* __restrict__ M,
                                                      float* __restrict__ W,
                                                      __nv_bfloat16* __restrict__ Wb) {
  constexpr int RT = D / 32, CT = D / 16;                 // 4 x 8 (D=128) or 2 x 4 (D=64)
  extern __shared__ __align__(16) float rb_sm[];
  float* Ys = rb_sm;
  float* Zs = Ys + D * D;
  float* Ts = Zs + D * D;
  __shared__ float s_c;
  __shared__ float s_red[16];
  const int h = blockIdx.x, tid = threadIdx.x;
  const float* Mh = M + static_cast<size_t>(h) * D * D;
  float* Wh = W + static_cast<size_t>(h) * D * D;
  {
    float t = 0.f;
    for (int i = tid; i < D * D; i += 512) t = fmaf(Mh[i], Mh[i], t);
    t = warp_sum(t);
    if (tid % 32 == 0) s_red[tid / 32] = t;
    __syncthreads();
    if (tid == 0) {
      float a = 0.f;
      for (int w = 0; w < 16; ++w) a += s_red[w];
      s_c = sqrtf(a);
    }
  }
  __syncthreads();
  const float c = s_c;
  __nv_bfloat16* Wbh = Wb + static_cast<size_t>(h) * D * D;
  if (!(c > 0.f) || !isfinite(c)) {
    for (int idx = tid; idx < D * D; idx += 512) {
      Wh[idx] = 0.f;
      Wbh[idx] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const float invc = 1.f / c;
  for (int idx = tid; idx < D * D; idx += 512) {
    Ys[idx] = Mh[idx] * invc;
    Zs[idx] = (idx / D == idx % D) ? 1.f : 0.f;
  }
  __syncthreads();
  const int r0 = (tid / 16) * RT, c0 = (tid % 16) * CT;
  auto mm = [&](const float* A, const float* B, float (&acc)[RT][CT]) {
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < CT; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      float a[RT], b[CT];
#pragma unroll
      for (int i = 0; i < RT; ++i) a[i] = A[(r0 + i) * D + k];
#pragma unroll
      for (int j = 0; j < CT; j += 4) {
        const float4 bv = *reinterpret_cast<const float4*>(&B[k * D + c0 + j]);
        b[j] = bv.x; b[j + 1] = bv.y; b[j + 2] = bv.z; b[j + 3] = bv.w;
      }
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < CT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  };
  float acc[RT][CT], acc2[RT][CT];
  for (int it = 0; it < kNsIters; ++it) {
    mm(Zs, Ys, acc);                                         // T = (3I - Z Y) / 2
    float dev = 0.f;
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < CT; ++j) {
        const float id = (r0 + i) == (c0 + j) ? 1.f : 0.f;
        dev = fmaxf(dev, fabsf(acc[i][j] - id));
        Ts[(r0 + i) * D + c0 + j] = 0.5f * (3.f * id - acc[i][j]);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
    if (tid % 32 == 0) s_red[tid / 32] = dev;
    __syncthreads();
    float mx = 0.f;
    for (int w = 0; w < 16; ++w) mx = fmaxf(mx, s_red[w]);
    if (mx < kNsTol) break;                                  // uniform: every thread sees mx
    __syncthreads();                                         // s_red is rewritten next step
    mm(Ys, Ts, acc);                                         // Y T
    mm(Ts, Zs, acc2);                                        // T Z
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int j = 0; j < CT; ++j) {
        Ys[(r0 + i) * D + c0 + j] = acc[i][j];
        Zs[(r0 + i) * D + c0 + j] = acc2[i][j];
      }
    __syncthreads();
  }
  const float sc = sqrtf(c);
  for (int idx = tid; idx < D * D; idx += 512) {
    Wh[idx] = Ys[idx] * sc;
    Wbh[idx] = __float2bfloat16_rn(Ys[idx] * sc);
  }
}

// ------------------------------------------------------------------ tensor-core whitening
// bf16 inputs with d = 128 take these two tcgen05 kernels instead of the CUDA-core ones.
// Tiles are 128 tokens x 128 dims, loaded by TMA with 128-byte swizzle (two 64-column atoms).

constexpr int kTcTile = 128 * 128 * 2;          // bytes of one bf16 tile
constexpr int kMomStages = 4;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
}

__device__ __forceinline__ bool rb_wait_quiet(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// part[h][p] = sum over the CTA's token tiles of Y^T Y: A = tile^T and B = tile, both read
// MN-major from the same shared-memory tile; the 128 x 128 fp32 sum stays in TMEM.
__global__ void __launch_bounds__(128) rb_moment_tc_kernel(const __grid_constant__ CUtensorMap map_y,
                                                           int tiles, float* __restrict__ part,
                                                           uint32_t* __restrict__ err,
                                                           uint64_t wait_ns) {
  extern __shared__ uint8_t rb_tc_raw[];
  uint8_t* st = align1024(rb_tc_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(st + kMomStages * kTcTile);
  uint64_t* empty = full + kMomStages;
  uint64_t* done = empty + kMomStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int p = blockIdx.x, P = gridDim.x, h = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
  const int t0 = static_cast<int>(static_cast<long long>(tiles) * p / P);
  const int T = static_cast<int>(static_cast<long long>(tiles) * (p + 1) / P) - t0;
  if (tid == 0) {
    for (int s = 0; s < kMomStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  if (tid == 0) {
    constexpr uint32_t idM = idesc_bf16(128, 128, true, true);
    tma_prefetch_desc(&map_y);
    int issued = 0;
    auto load = [&](int t) {
      const int s = t % kMomStages;
      mbar_arrive_expect_tx(&full[s], kTcTile);
      for (int a = 0; a < 2; ++a)
        tma_load_3d(st + s * kTcTile + a * 16384, &map_y, &full[s], a * 64, (t0 + t) * 128, h);
      issued = t + 1;
    };
    for (int t = 0; t < min(T, kMomStages); ++t) load(t);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % kMomStages;
      if (!mbar_wait(&full[s], (t / kMomStages) & 1, abort_flag, err, wait_ns)) { ok = false; break; }
      tc_fence_after_sync();
      const uint64_t d0 = sdesc_sw128(smem_u32(st + s * kTcTile), 16384, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t dk = d0 + static_cast<uint64_t>((kk * 2048) >> 4);
        mma_ss(tbase, dk, dk, idM, (t > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&empty[s]);
      if (t + kMomStages < T) {
        if (!mbar_wait(&empty[s], (t / kMomStages) & 1, abort_flag, err, wait_ns)) { ok = false; break; }
        load(t + kMomStages);
      }
    }
    if (!ok)                                               // drain the loads still in flight
      for (int t = max(0, issued - kMomStages); t < issued; ++t)
        rb_wait_quiet(&full[t % kMomStages], (t / kMomStages) & 1);
    tc_commit(done);
    rb_wait_quiet(done, 0);
  }
  __syncthreads();
  const bool fine = !*abort_flag;
  tc_fence_after_sync();
  float* out = part + (static_cast<size_t>(h) * P + p) * 128 * 128;
  const int row = warp * 32 + (tid % 32);
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t r[32];
    if (T > 0 && fine) {
      tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + cc * 32, r);
    } else {
      for (int j = 0; j < 32; ++j) r[j] = 0u;
    }
    float4* dst = reinterpret_cast<float4*>(out + row * 128 + cc * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                           __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 128);
  }
}

// X rows = bf16(unit(W y)) for the CTA's token tiles: A = Y tile and B = W (both K-major), two
// TMEM accumulators; warps 0-3 normalise and store one row per thread while warp 4 (one
// thread) loads and issues the next tile.
__global__ void __launch_bounds__(160) rb_whiten_tc_kernel(const __grid_constant__ CUtensorMap map_y,
                                                           const __grid_constant__ CUtensorMap map_w,
                                                           int N, int tiles,
                                                           __nv_bfloat16* __restrict__ X,
                                                           uint32_t* __restrict__ err,
                                                           uint64_t wait_ns) {
  extern __shared__ uint8_t rb_tc_raw[];
  uint8_t* wst = align1024(rb_tc_raw);
  uint8_t* yst = wst + kTcTile;                          // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(yst + 2 * kTcTile);
  uint64_t* wfull = bars;
  uint64_t* yfull = bars + 1;                            // [2]
  uint64_t* yempty = bars + 3;                           // [2]
  uint64_t* accfull = bars + 5;                          // [2]
  uint64_t* accempty = bars + 7;                         // [2], count 128
  uint64_t* done = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int h = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
  const int t0 = static_cast<int>(static_cast<long long>(tiles) * blockIdx.x / gridDim.x);
  const int T = static_cast<int>(static_cast<long long>(tiles) * (blockIdx.x + 1) / gridDim.x) - t0;
  if (tid == 0) {
    mbar_init(wfull, 1);
    mbar_init(done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&yfull[b], 1);
      mbar_init(&yempty[b], 1);
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 128);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  if (warp == 4) {
    if ((tid % 32) == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      tma_prefetch_desc(&map_y);
      tma_prefetch_desc(&map_w);
      mbar_arrive_expect_tx(wfull, kTcTile);
      for (int a = 0; a < 2; ++a) tma_load_3d(wst + a * 16384, &map_w, wfull, a * 64, 0, h);
      int issued = 0;
      auto load = [&](int t) {
        const int s = t & 1;
        mbar_arrive_expect_tx(&yfull[s], kTcTile);
        for (int a = 0; a < 2; ++a)
          tma_load_3d(yst + s * kTcTile + a * 16384, &map_y, &yfull[s], a * 64, (t0 + t) * 128, h);
        issued = t + 1;
      };
      for (int t = 0; t < min(T, 2); ++t) load(t);
      bool ok = mbar_wait(wfull, 0, abort_flag, err, wait_ns);
      const uint64_t wd = sdesc_sw128(smem_u32(wst), 16, 1024);
      for (int t = 0; ok && t < T; ++t) {
        const int s = t & 1;
        if (!mbar_wait(&yfull[s], (t >> 1) & 1, abort_flag, err, wait_ns)) { ok = false; break; }
        if (t >= 2 && !mbar_wait(&accempty[s], ((t >> 1) - 1) & 1, abort_flag, err, wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint64_t yd = sdesc_sw128(smem_u32(yst + s * kTcTile), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk / 4) * 16384 + (kk % 4) * 32) / 16;
          mma_ss(tbase + s * 128, yd + off, wd + off, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&accfull[s]);
        tc_commit(&yempty[s]);
        if (t + 2 < T) {
          if (!mbar_wait(&yempty[s], (t >> 1) & 1, abort_flag, err, wait_ns)) { ok = false; break; }
          load(t + 2);
        }
      }
      if (!ok) {
        for (int t = max(0, issued - 2); t < issued; ++t) rb_wait_quiet(&yfull[t & 1], (t >> 1) & 1);
        rb_wait_quiet(wfull, 0);
      }
      tc_commit(done);                                     // no MMA left in flight before TMEM
      rb_wait_quiet(done, 0);                              // is freed
    }
  } else {
    const int row = tid;                                 // TMEM lane = token row of the tile
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&accfull[b], (t >> 1) & 1, abort_flag, err, wait_ns));
      if (!got) break;
      tc_fence_after_sync();
      float v[128];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + b * 128 + cc * 32, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[cc * 32 + j] = __uint_as_float(r[j]);
      }
      tc_fence_before_sync();
      mbar_arrive(&accempty[b]);                         // accumulator b may be reused
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 128; ++j) ss = fmaf(v[j], v[j], ss);
      const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
      const int tok = (t0 + t) * 128 + row;
      if (tok < N) {
        uint4* dst = reinterpret_cast<uint4*>(X + (static_cast<size_t>(h) * N + tok) * 128);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          dst[q] = make_uint4(pack_bf16(v[8 * q] * inv, v[8 * q + 1] * inv),
                              pack_bf16(v[8 * q + 2] * inv, v[8 * q + 3] * inv),
                              pack_bf16(v[8 * q + 4] * inv, v[8 * q + 5] * inv),
                              pack_bf16(v[8 * q + 6] * inv, v[8 * q + 7] * inv));
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 256);
  }
}

// ------------------------------------------------------------------ whitening
// X[h][i] = bf16(W y_i / |W y_i|) (0 for a zero vector).  W^T in shared memory; a warp
// transforms 8 tokens at once, lane l owning outputs l, l+32, ...
template <int D, typename T>
__global__ void __launch_bounds__(kRbThreads) rb_whiten_kernel(const T* __restrict__ Y,
                                                               const float* __restrict__ W,
                                                               int N,
                                                               __nv_bfloat16* __restrict__ X) {
  constexpr int R = D / 32;
  constexpr int G = 8;                                     // tokens per warp step
  extern __shared__ __align__(16) float rb_sm[];
  float* Wt = rb_sm;                                       // [D][D]: Wt[e][o] = W[o][e]
  float* qs = Wt + D * D;                                  // [warps][G][D]
  const int h = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float* Wh = W + static_cast<size_t>(h) * D * D;
  for (int idx = threadIdx.x; idx < D * D; idx += kRbThreads) {
    const int o = idx / D, e = idx % D;
    Wt[e * D + o] = Wh[idx];
  }
  __syncthreads();
  float* q = qs + warp * G * D;
  const int tok_per_cta = kRbWarps * G * 4;
  const int t_begin = blockIdx.x * tok_per_cta;
  const T* Yh = Y + static_cast<size_t>(h) * N * D;
  __nv_bfloat16* Xh = X + static_cast<size_t>(h) * N * D;
  for (int g0 = t_begin + warp * G; g0 < min(N, t_begin + tok_per_cta); g0 += kRbWarps * G) {
    const int ng = min(G, N - g0);
    __syncwarp();
    for (int i = lane; i < G * D; i += 32) {
      const int t = i / D, e = i % D;
      q[i] = t < ng ? ld_f(Yh + static_cast<size_t>(g0 + t) * D + e) : 0.f;
    }
    __syncwarp();
    float acc[G][R];
#pragma unroll
    for (int t = 0; t < G; ++t)
#pragma unroll
      for (int j = 0; j < R; ++j) acc[t][j] = 0.f;
#pragma unroll 2
    for (int e = 0; e < D; e += 4) {
      float w[4][R];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < R; ++j) w[u][j] = Wt[(e + u) * D + lane + 32 * j];
#pragma unroll
      for (int t = 0; t < G; ++t) {
        const float4 qv = *reinterpret_cast<const float4*>(&q[t * D + e]);
        const float qq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int j = 0; j < R; ++j) acc[t][j] = fmaf(w[u][j], qq[u], acc[t][j]);
      }
    }
#pragma unroll
    for (int t = 0; t < G; ++t) {
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < R; ++j) ss = fmaf(acc[t][j], acc[t][j], ss);
      ss = warp_sum(ss);
      const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
      if (t < ng) {
#pragma unroll
        for (int j = 0; j < R; ++j)
          Xh[static_cast<size_t>(g0 + t) * D + lane + 32 * j] = __float2bfloat16_rn(acc[t][j] * inv);
      }
    }
  }
}

// ------------------------------------------------------------------ one level
// Level metadata (identical for every head): nodes[g] = (start, mid, end, chunk0) in token
// positions, with one sentinel node whose chunk0 is the level's chunk count; chunks[c] =
// (node, start, end, 0).

// Lanes per token in the level passes: lane group g of a warp handles one token, lane s of
// the group the DPL = D / 8 dimensions [s*DPL, (s+1)*DPL) of it (two or one 16-byte loads).
constexpr int kLanesPerTok = 8;
constexpr int kTokPerWarp = 32 / kLanesPerTok;

template <int DPL>
__device__ __forceinline__ void load_dims(const __nv_bfloat16* p, uint32_t (&w)[DPL / 2]) {
#pragma unroll
  for (int q = 0; q < DPL / 8; ++q)
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[4 * q]), "=r"(w[4 * q + 1]), "=r"(w[4 * q + 2]), "=r"(w[4 * q + 3])
                 : "l"(p + 8 * q));
}

template <int DPL>
__device__ __forceinline__ float group_dot(const uint32_t (&w)[DPL / 2], const float (&v)[DPL],
                                           float (&x)[DPL]) {
  float y = 0.f;
#pragma unroll
  for (int i = 0; i < DPL / 2; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    y = fmaf(x[2 * i], v[2 * i], y);
    y = fmaf(x[2 * i + 1], v[2 * i + 1], y);
  }
#pragma unroll
  for (int o = 1; o < kLanesPerTok; o <<= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
  return y;
}

// Pass over a chunk: sum of (x.v) x (and of x on the first pass).  Tokens are taken in a
// fixed order (warp, step, group) and the partial sums are reduced over groups and then
// warps in a fixed order.
template <int D, bool kFirst>
__global__ void __launch_bounds__(kRbThreads, 3) rb_power_kernel(
    const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm, int N,
    const int4* __restrict__ chunks, int nch, const float* __restrict__ vnode, int nnodes,
    float* __restrict__ part) {
  constexpr int DPL = D / kLanesPerTok;
  constexpr int U = kRowsInFlight / 2;                     // steps of 4 tokens in flight
  __shared__ float red[kRbWarps][2 * D];
  __shared__ int toks[kChunk];                             // the chunk's token ids, staged once
  const int c = blockIdx.x, h = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int grp = lane / kLanesPerTok, sub = lane % kLanesPerTok;
  const int4 ch = chunks[c];
  for (int i = threadIdx.x; i < ch.z - ch.y; i += kRbThreads)
    toks[i] = min(max(perm[static_cast<size_t>(h) * N + ch.y + i], 0), N - 1);
  float v[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j)
    v[j] = kFirst ? rsqrtf(static_cast<float>(D))
                  : vnode[(static_cast<size_t>(h) * nnodes + ch.x) * D + sub * DPL + j];
  __syncthreads();
  float sxv[DPL], sx[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) sxv[j] = sx[j] = 0.f;
  const __nv_bfloat16* Xh = X + static_cast<size_t>(h) * N * D + sub * DPL;
  for (int p0 = ch.y + warp * kTokPerWarp * U; p0 < ch.z; p0 += kRbWarps * kTokPerWarp * U) {
    uint32_t raw[U][DPL / 2];
#pragma unroll
    for (int u = 0; u < U; ++u) {                          // U x 4 row loads in flight
      const int pos = min(p0 + u * kTokPerWarp + grp, ch.z - 1);
      load_dims<DPL>(Xh + static_cast<size_t>(toks[pos - ch.y]) * D, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float x[DPL];
      const float y = group_dot<DPL>(raw[u], v, x);
      if (p0 + u * kTokPerWarp + grp < ch.z) {
#pragma unroll
        for (int j = 0; j < DPL; ++j) {
          sxv[j] = fmaf(y, x[j], sxv[j]);
          if (kFirst) sx[j] += x[j];
        }
      }
    }
  }
  // groups -> lanes 0..7 of the warp, in a fixed order
#pragma unroll
  for (int o = kLanesPerTok; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      sxv[j] += __shfl_xor_sync(0xffffffffu, sxv[j], o);
      if (kFirst) sx[j] += __shfl_xor_sync(0xffffffffu, sx[j], o);
    }
  if (grp == 0) {
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      red[warp][sub * DPL + j] = sxv[j];
      red[warp][D + sub * DPL + j] = sx[j];
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < (kFirst ? 2 * D : D); t += kRbThreads) {
    float s = 0.f;
    for (int w = 0; w < kRbWarps; ++w) s += red[w][t];
    part[(static_cast<size_t>(h) * nch + c) * 2 * D + t] = s;
  }
}

// Per node: mu (first pass), w = S/n - (mu.v) mu, v <- w / |w| (kept if |w| = 0).
template <int D, bool kFirst>
__global__ void __launch_bounds__(D) rb_node_reduce_kernel(const float* __restrict__ part,
                                                           int nch,
                                                           const int4* __restrict__ nodes,
                                                           int nnodes, float* __restrict__ mu,
                                                           float* __restrict__ vnode) {
  __shared__ float red[D / 32];
  __shared__ float s_val;
  const int g = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  const int4 nd = nodes[g];
  const int c_end = nodes[g + 1].w;
  const float n = static_cast<float>(nd.z - nd.x);
  float S = 0.f, Sx = 0.f;
  for (int c = nd.w; c < c_end; ++c) {
    const float* pc = part + (static_cast<size_t>(h) * nch + c) * 2 * D;
    S += pc[t];
    if (kFirst) Sx += pc[D + t];
  }
  const size_t at = (static_cast<size_t>(h) * nnodes + g) * D + t;
  const float m = kFirst ? Sx / n : mu[at];
  if (kFirst) mu[at] = m;
  const float vp = kFirst ? rsqrtf(static_cast<float>(D)) : vnode[at];
  auto block_sum = [&](float x) {
    x = warp_sum(x);
    __syncthreads();
    if (t % 32 == 0) red[t / 32] = x;
    __syncthreads();
    if (t == 0) {
      float s = 0.f;
      for (int i = 0; i < D / 32; ++i) s += red[i];
      s_val = s;
    }
    __syncthreads();
    return s_val;
  };
  const float muv = block_sum(m * vp);
  const float w = S / n - muv * m;
  const float nrm2 = block_sum(w * w);
  vnode[at] = nrm2 > 0.f ? w * rsqrtf(nrm2) : vp;
}

// keys[pos] = order key of x.v (the order of (x - mu).v), and the histogram of the top byte.
template <int D>
__global__ void __launch_bounds__(kRbThreads, 3) rb_project_kernel(
    const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm, int N,
    const int4* __restrict__ chunks, const float* __restrict__ vnode, int nnodes,
    uint32_t* __restrict__ keys, uint32_t* __restrict__ hist) {
  constexpr int DPL = D / kLanesPerTok;
  constexpr int U = kRowsInFlight / 2;
  __shared__ uint32_t sh[256];
  __shared__ int toks[kChunk];
  const int c = blockIdx.x, h = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int grp = lane / kLanesPerTok, sub = lane % kLanesPerTok;
  const int4 ch = chunks[c];
  sh[threadIdx.x] = 0u;
  for (int i = threadIdx.x; i < ch.z - ch.y; i += kRbThreads)
    toks[i] = min(max(perm[static_cast<size_t>(h) * N + ch.y + i], 0), N - 1);
  float v[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j)
    v[j] = vnode[(static_cast<size_t>(h) * nnodes + ch.x) * D + sub * DPL + j];
  __syncthreads();
  const __nv_bfloat16* Xh = X + static_cast<size_t>(h) * N * D + sub * DPL;
  for (int p0 = ch.y + warp * kTokPerWarp * U; p0 < ch.z; p0 += kRbWarps * kTokPerWarp * U) {
    uint32_t raw[U][DPL / 2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int pos = min(p0 + u * kTokPerWarp + grp, ch.z - 1);
      load_dims<DPL>(Xh + static_cast<size_t>(toks[pos - ch.y]) * D, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float x[DPL];
      const float y = group_dot<DPL>(raw[u], v, x);
      const int pos = p0 + u * kTokPerWarp + grp;
      if (sub == 0 && pos < ch.z) {
        const uint32_t key = rb_order_key(y);
        keys[static_cast<size_t>(h) * N + pos] = key;
        atomicAdd(&sh[key >> 24], 1u);
      }
    }
  }
  __syncthreads();
  const uint32_t cnt = sh[threadIdx.x];
  if (cnt) atomicAdd(&hist[(static_cast<size_t>(h) * nnodes + ch.x) * 256 + threadIdx.x], cnt);
}

// One radix digit per node: the largest digit x with count(digit >= x) >= need among the
// keys matching the prefix; state = (prefix, need); the histogram is cleared for the next pass.
__global__ void __launch_bounds__(32) rb_pick_kernel(uint32_t* __restrict__ hist,
                                                     const int4* __restrict__ nodes, int nnodes,
                                                     uint32_t* __restrict__ state, int shift) {
  const int g = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const size_t ng = static_cast<size_t>(h) * nnodes + g;
  uint32_t* hb = hist + ng * 256;
  const int4 nd = nodes[g];
  uint32_t prefix = shift == 24 ? 0u : state[ng * 2];
  int need = shift == 24 ? (nd.y - nd.x) : static_cast<int>(state[ng * 2 + 1]);
  uint32_t cnt[8], local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    cnt[j] = hb[lane * 8 + j];
    local += cnt[j];
    hb[lane * 8 + j] = 0u;
  }
  uint32_t suf = local;                                   // inclusive suffix sum over lanes
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += o;
  }
  uint32_t above = suf - local;
  int best = -1;
  uint32_t best_gt = 0;
#pragma unroll
  for (int j = 7; j >= 0; --j) {
    const uint32_t ge = above + cnt[j];
    if (best < 0 && ge >= static_cast<uint32_t>(need)) {
      best = lane * 8 + j;
      best_gt = above;
    }
    above = ge;
  }
  const int dd = __reduce_max_sync(0xffffffffu, best);
  const uint32_t gt = __shfl_sync(0xffffffffu, best_gt, max(dd, 0) / 8);
  if (lane == 0) {
    if (dd >= 0) {
      need -= static_cast<int>(gt);
      prefix |= static_cast<uint32_t>(dd) << shift;
    }
    state[ng * 2] = prefix;
    state[ng * 2 + 1] = static_cast<uint32_t>(need);
  }
}

// Histogram of the digit at `shift` of the keys that match the node's prefix so far.
__global__ void __launch_bounds__(kRbThreads) rb_hist_kernel(const uint32_t* __restrict__ keys,
                                                             int N, const int4* __restrict__ chunks,
                                                             const uint32_t* __restrict__ state,
                                                             int nnodes,
                                                             uint32_t* __restrict__ hist,
                                                             int shift) {
  __shared__ uint32_t sh[256];
  const int c = blockIdx.x, h = blockIdx.y;
  const int4 ch = chunks[c];
  sh[threadIdx.x] = 0u;
  const size_t ng = static_cast<size_t>(h) * nnodes + ch.x;
  const uint32_t prefix = state[ng * 2];
  const uint32_t mask = 0xFFFFFFFFu << (shift + 8);
  __syncthreads();
  for (int pos = ch.y + threadIdx.x; pos < ch.z; pos += kRbThreads) {
    const uint32_t key = keys[static_cast<size_t>(h) * N + pos];
    if ((key & mask) == prefix) atomicAdd(&sh[(key >> shift) & 255u], 1u);
  }
  __syncthreads();
  const uint32_t cnt = sh[threadIdx.x];
  if (cnt) atomicAdd(&hist[ng * 256 + threadIdx.x], cnt);
}

// Per chunk: keys above the threshold and keys equal to it.
__global__ void __launch_bounds__(kRbThreads) rb_count_kernel(const uint32_t* __restrict__ keys,
                                                              int N,
                                                              const int4* __restrict__ chunks,
                                                              int nch,
                                                              const uint32_t* __restrict__ state,
                                                              int nnodes,
                                                              int* __restrict__ cnt) {
  __shared__ int s_gt[kRbWarps], s_eq[kRbWarps];
  const int c = blockIdx.x, h = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int4 ch = chunks[c];
  const uint32_t T = state[(static_cast<size_t>(h) * nnodes + ch.x) * 2];
  int gt = 0, eq = 0;
  for (int pos = ch.y + threadIdx.x; pos < ch.z; pos += kRbThreads) {
    const uint32_t key = keys[static_cast<size_t>(h) * N + pos];
    gt += key > T;
    eq += key == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    s_gt[warp] = gt;
    s_eq[warp] = eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < kRbWarps; ++w) {
      a += s_gt[w];
      b += s_eq[w];
    }
    cnt[(static_cast<size_t>(h) * nch + c) * 2] = a;
    cnt[(static_cast<size_t>(h) * nch + c) * 2 + 1] = b;
  }
}

// Per node, over its chunks in order: equal keys, left and right tokens before each chunk.
__global__ void __launch_bounds__(32) rb_scan_kernel(const int* __restrict__ cnt, int nch,
                                                     const int4* __restrict__ nodes, int nnodes,
                                                     const int4* __restrict__ chunks,
                                                     const uint32_t* __restrict__ state,
                                                     int* __restrict__ base) {
  const int g = blockIdx.x, h = blockIdx.y;
  if (threadIdx.x != 0) return;
  const int4 nd = nodes[g];
  const int c_end = nodes[g + 1].w;
  const int need = static_cast<int>(state[(static_cast<size_t>(h) * nnodes + g) * 2 + 1]);
  int eq_before = 0, left_before = 0, right_before = 0;
  for (int c = nd.w; c < c_end; ++c) {
    const size_t hc = static_cast<size_t>(h) * nch + c;
    const int gt = cnt[hc * 2], eq = cnt[hc * 2 + 1];
    const int size = chunks[c].z - chunks[c].y;
    const int left = gt + min(max(need - eq_before, 0), eq);
    base[hc * 3] = eq_before;
    base[hc * 3 + 1] = left_before;
    base[hc * 3 + 2] = right_before;
    eq_before += eq;
    left_before += left;
    right_before += size - left;
  }
}

// Stable two-way partition of the chunk's tokens: left if key > T, or key == T and the
// token is among the first `need` equal keys of the node (in position order).
__global__ void __launch_bounds__(kRbThreads) rb_scatter_kernel(
    const uint32_t* __restrict__ keys, const int32_t* __restrict__ perm_in, int N,
    const int4* __restrict__ chunks, int nch, const int4* __restrict__ nodes,
    const uint32_t* __restrict__ state, int nnodes, const int* __restrict__ base,
    int32_t* __restrict__ perm_out) {
  __shared__ int s_eq[kRbWarps], s_left[kRbWarps];
  const int c = blockIdx.x, h = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int4 ch = chunks[c];
  const int4 nd = nodes[ch.x];
  const size_t ng = static_cast<size_t>(h) * nnodes + ch.x;
  const uint32_t T = state[ng * 2];
  const int need = static_cast<int>(state[ng * 2 + 1]);
  const size_t hc = static_cast<size_t>(h) * nch + c;
  int eq_before = base[hc * 3], left_before = base[hc * 3 + 1], right_before = base[hc * 3 + 2];
  const uint32_t lt = (1u << lane) - 1u;
  for (int r0 = ch.y; r0 < ch.z; r0 += kRbThreads) {
    const int pos = r0 + threadIdx.x;
    const bool valid = pos < ch.z;
    const uint32_t key = valid ? keys[static_cast<size_t>(h) * N + pos] : 0u;
    const bool eq = valid && key == T;
    // exclusive rank of the equal keys in this round
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_eq[warp] = __popc(be);
    __syncthreads();
    int eq_off = 0, eq_tot = 0;
    for (int w = 0; w < kRbWarps; ++w) {
      if (w < warp) eq_off += s_eq[w];
      eq_tot += s_eq[w];
    }
    const int eq_rank = eq_before + eq_off + __popc(be & lt);
    const bool left = valid && (key > T || (eq && eq_rank < need));
    const uint32_t bl = __ballot_sync(0xffffffffu, left);
    if (lane == 0) s_left[warp] = __popc(bl);
    __syncthreads();
    int l_off = 0, l_tot = 0;
    for (int w = 0; w < kRbWarps; ++w) {
      if (w < warp) l_off += s_left[w];
      l_tot += s_left[w];
    }
    const int left_rank = l_off + __popc(bl & lt);
    if (valid) {
      const int dst = left ? nd.x + left_before + left_rank
                           : nd.y + right_before + (static_cast<int>(threadIdx.x) - left_rank);
      // the counts make dst fall inside the node's child; the guard keeps a bad count local
      if (dst >= (left ? nd.x : nd.y) && dst < (left ? nd.y : nd.z))
        perm_out[static_cast<size_t>(h) * N + dst] = perm_in[static_cast<size_t>(h) * N + pos];
    }
    const int nvalid = min(kRbThreads, ch.z - r0);
    eq_before += eq_tot;
    left_before += l_tot;
    right_before += nvalid - l_tot;
    __syncthreads();                                       // s_eq / s_left reused next round
  }
}

// ------------------------------------------------------------------ tensor-core node moments
// Levels whose nodes hold at least kCovMinNode tokens (d = 128): instead of kPowerIters passes
// over the rows, one pass gathers each chunk's rows (by the permutation) into shared memory
// and sums x x^T on the tensor cores (both operands the MN-major tile, as in rb_moment_tc),
// plus the sum of x; rb_cov_node then runs the power iterations on the node's 128 x 128
// matrix: v <- (S/n - mu mu^T) v, the same update as the row passes.

constexpr int kCovChunk = 16384;      // tokens per CTA of the moment pass
constexpr int kCovMinNode = 256;     // smallest node size that takes this path
constexpr int kCovStride = 128 * 128 + 128;   // floats per partial: x x^T, then sum x

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The power iterations of one node from its second moment S (shared memory, [128][128]) and
// column sums sxv (thread t: dimension t), 128 threads: mu = sum x / n, then kPowerIters steps
// v <- w / |w|, w = S v / n - (mu . v) mu, from v0 = (1,...,1)/sqrt(d).  Writes mu and v of
// node g.  Shared by rb_cov_node_kernel and the single-chunk form of rb_cov_tc_kernel, so both
// take the same arithmetic.
__device__ __forceinline__ void rb_node_power(const float* Ssm, float sxv, float n, int t,
                                              float* vs, float* red, float* s_val, int h, int g,
                                              int nnodes, float* __restrict__ mu,
                                              float* __restrict__ vnode) {
  const float m = sxv / n;
  float v = rsqrtf(128.f);
  auto block_sum = [&](float x) {
    x = warp_sum(x);
    __syncthreads();
    if (t % 32 == 0) red[t / 32] = x;
    __syncthreads();
    if (t == 0) *s_val = red[0] + red[1] + red[2] + red[3];
    __syncthreads();
    return *s_val;
  };
  for (int it = 0; it < kPowerIters; ++it) {
    vs[t] = v;
    __syncthreads();
    float sv = 0.f;
    for (int j = 0; j < 128; ++j) sv = fmaf(Ssm[j * 128 + t], vs[j], sv);   // S symmetric
    const float muv = block_sum(m * v);
    const float w = sv / n - muv * m;
    const float nrm2 = block_sum(w * w);
    v = nrm2 > 0.f ? w * rsqrtf(nrm2) : v;
  }
  const size_t at = (static_cast<size_t>(h) * nnodes + g) * 128 + t;
  mu[at] = m;
  vnode[at] = v;
}

// One chunk of a node: rows gathered by the permutation into 128-token tiles (cp.async, each
// 16-byte piece written to its place in the 128-byte swizzled layout, zero past the chunk
// end), the next tile in flight while the tensor core consumes the current one.  kSingle: every
// node of the level is one chunk, so the CTA holds the node's whole second moment and runs its
// power iterations itself (mu, v of the node) instead of writing the 66 KB partial for
// rb_cov_node_kernel.
template <bool kSingle>
__global__ void __launch_bounds__(128) rb_cov_tc_kernel(const __nv_bfloat16* __restrict__ X,
                                                        const int32_t* __restrict__ perm, int N,
                                                        const int4* __restrict__ cchunks,
                                                        int ncch, float* __restrict__ cpart,
                                                        uint32_t* __restrict__ err,
                                                        uint64_t wait_ns, int nnodes,
                                                        float* __restrict__ mu,
                                                        float* __restrict__ vnode) {
  extern __shared__ uint8_t rb_tc_raw[];
  uint8_t* st = align1024(rb_tc_raw);                    // 2 stages x 32 KB
  uint64_t* mdone = reinterpret_cast<uint64_t*>(st + 2 * kTcTile);   // [2]
  uint64_t* done = mdone + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* toks = reinterpret_cast<int*>(tmem_slot + 4);     // [2][128] token ids of a tile
  float* red = reinterpret_cast<float*>(toks + 256);     // [128][8] column sums
  const int c = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
  const int4 ch = cchunks[c];
  const int T = (ch.z - ch.y + 127) / 128;
  const int cidx = tid % 16;                             // this thread's 16-byte column chunk
  if (tid == 0) {
    mbar_init(&mdone[0], 1);
    mbar_init(&mdone[1], 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  const int32_t* ph = perm + static_cast<size_t>(h) * N;
  const __nv_bfloat16* Xh = X + static_cast<size_t>(h) * N * 128;
  auto stage_toks = [&](int t) {                         // thread tid: row tid of tile t
    const int pos = ch.y + t * 128 + tid;
    toks[(t & 1) * 128 + tid] = pos < ch.z ? min(max(ph[pos], 0), N - 1) : -1;
  };
  auto issue_tile = [&](int t) {                         // after toks of tile t are visible
    uint8_t* tile = st + (t & 1) * kTcTile;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = (tid + 128 * i) >> 4;
      const int tok = toks[(t & 1) * 128 + r];
      cp_async16_zfill(tile + (cidx / 8) * 16384 + r * 128 + (((cidx % 8) ^ (r & 7)) * 16),
                       Xh + static_cast<size_t>(tok < 0 ? 0 : tok) * 128 + cidx * 8, tok >= 0);
    }
    cp_async_commit();
  };
  if (T > 0) stage_toks(0);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  constexpr uint32_t idM = idesc_bf16(128, 128, true, true);
  float sx[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) sx[j] = 0.f;
  if (T > 0) issue_tile(0);
  bool ok = true;
  for (int t = 0; t < T; ++t) {
    const int s = t & 1;
    if (t + 1 < T) stage_toks(t + 1);                    // its latency overlaps the wait below
    cp_async_wait_all();                                 // this thread's pieces of tile t
    fence_proxy_async_smem();                            // visible to the tensor core
    __syncthreads();                                     // everyone's pieces, and toks(t+1)
    const uint8_t* tile = st + s * kTcTile;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = (tid + 128 * i) >> 4;
      const uint4 u = *reinterpret_cast<const uint4*>(
          tile + (cidx / 8) * 16384 + r * 128 + (((cidx % 8) ^ (r & 7)) * 16));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        sx[2 * q] += __uint_as_float(w[q] << 16);
        sx[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
      }
    }
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t d0 = sdesc_sw128(smem_u32(tile), 16384, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t dk = d0 + static_cast<uint64_t>((kk * 2048) >> 4);
        mma_ss(tbase, dk, dk, idM, (t > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&mdone[s]);
    }
    if (t + 1 < T) {
      // stage s^1 held tile t-1: its MMAs must be done before it is overwritten
      if (t >= 1)
        ok = __syncthreads_and(mbar_wait(&mdone[s ^ 1], ((t - 1) >> 1) & 1, abort_flag, err, wait_ns));
      if (!ok) break;
      issue_tile(t + 1);
    }
  }
  cp_async_wait_all();                                   // nothing of ours left in flight
  if (tid == 0) {
    tc_commit(done);                                     // every MMA issued has completed
    rb_wait_quiet(done, 0);
  }
  __syncthreads();
  const bool fine = ok && !*abort_flag;
  tc_fence_after_sync();
  const int row = warp * 32 + (tid % 32);
  if constexpr (kSingle) {
    // S from TMEM into the (now idle) tile stages, the column sums in thread order, then the
    // power iterations - the values rb_cov_node_kernel would read back from the partial
    float* Ssm = reinterpret_cast<float*>(st);          // [128][128] = both 32 KB stages
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      if (fine) {
        tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + cc * 32, r);
      } else {
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      }
      float4* dst = reinterpret_cast<float4*>(Ssm + row * 128 + cc * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) red[tid * 8 + j] = sx[j];
    __syncthreads();
    float sxv = 0.f;
    {
      const int dim = tid, cc = dim / 8, j = dim % 8;
      float a = 0.f;
      for (int g = 0; g < 8; ++g) a += red[(g * 16 + cc) * 8 + j];
      sxv = 0.f + (fine ? a : 0.f);                     // the node's sum over its one chunk
    }
    __shared__ float vs[128], pred[4], s_val;
    rb_node_power(Ssm, sxv, static_cast<float>(ch.z - ch.y), tid, vs, pred, &s_val, h, ch.x,
                  nnodes, mu, vnode);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after_sync();
      tmem_dealloc(tbase, 128);
    }
    return;
  }
  float* out = cpart + (static_cast<size_t>(h) * ncch + c) * kCovStride;
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t r[32];
    if (fine) {
      tmem_ld32(tbase + (static_cast<uint32_t>(warp * 32) << 16) + cc * 32, r);
    } else {
      for (int j = 0; j < 32; ++j) r[j] = 0u;
    }
    float4* dst = reinterpret_cast<float4*>(out + row * 128 + cc * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                           __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
  }
  // column sums: the 8 threads with the same chunk index, in thread order
#pragma unroll
  for (int j = 0; j < 8; ++j) red[tid * 8 + j] = sx[j];
  __syncthreads();
  {
    const int dim = tid, cc = dim / 8, j = dim % 8;
    float a = 0.f;
    for (int g = 0; g < 8; ++g) a += red[(g * 16 + cc) * 8 + j];
    out[128 * 128 + dim] = fine ? a : 0.f;
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 128);
  }
}

// Per node: S = sum of the chunk partials (in order), mu = sum x / n, then kPowerIters steps
// v <- w / |w|, w = S v / n - (mu . v) mu, from v0 = (1,...,1)/sqrt(d).
__global__ void __launch_bounds__(128) rb_cov_node_kernel(const float* __restrict__ cpart,
                                                          int ncch,
                                                          const int4* __restrict__ cnodes,
                                                          const int4* __restrict__ nodes,
                                                          int nnodes, float* __restrict__ mu,
                                                          float* __restrict__ vnode) {
  extern __shared__ __align__(16) float Ssm[];           // [128][128]
  __shared__ float vs[128];
  __shared__ float red[4];
  __shared__ float s_val;
  const int g = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  const int4 cn = cnodes[g];
  const int4 nd = nodes[g];
  const float n = static_cast<float>(nd.z - nd.x);
  for (int row0 = 0; row0 < 128; row0 += 8) {
    float a[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) a[r] = 0.f;
    for (int c = cn.x; c < cn.y; ++c) {
      const float* pc = cpart + (static_cast<size_t>(h) * ncch + c) * kCovStride + t;
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] += pc[(row0 + r) * 128];   // 8 rows in flight
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) Ssm[(row0 + r) * 128 + t] = a[r];
  }
  float sxv = 0.f;
  for (int c = cn.x; c < cn.y; ++c) sxv += cpart[(static_cast<size_t>(h) * ncch + c) * kCovStride + 128 * 128 + t];
  rb_node_power(Ssm, sxv, n, t, vs, red, &s_val, h, g, nnodes, mu, vnode);
}

// ------------------------------------------------------------------ host side

namespace {

struct LevelMeta {
  int node_off, nnodes;      // into the int4 node array (nnodes + 1 entries incl. sentinel)
  int chunk_off, nch;        // into the int4 chunk array
  bool cov;                  // every node >= kCovMinNode tokens: tensor-core moments
  int cnode_off, cchunk_off, ncch;   // per node (first, end) moment chunk; moment chunks
};

struct Plan {
  int nb = 0;
  std::vector<LevelMeta> levels;
  std::vector<int4> nodes, chunks, cnodes, cchunks;
  int max_nodes = 0, max_chunks = 0, max_cchunks = 0;
};

Plan make_plan(int N, int block) {
  Plan P;
  P.nb = (N + block - 1) / block;
  auto off = [&](int b) { return b >= P.nb ? N : b * block; };
  std::vector<std::pair<int, int>> frontier{{0, P.nb}};
  while (!frontier.empty()) {
    std::vector<std::pair<int, int>> next;
    LevelMeta L{static_cast<int>(P.nodes.size()), 0, static_cast<int>(P.chunks.size()), 0,
                true, static_cast<int>(P.cnodes.size()), static_cast<int>(P.cchunks.size()), 0};
    for (auto [lo, hi] : frontier) {
      if (hi - lo < 2) continue;
      const int mid = lo + (hi - lo + 1) / 2;
      const int a = off(lo), m = off(mid), e = off(hi);
      P.nodes.push_back(make_int4(a, m, e, L.nch));
      for (int s = a; s < e; s += kChunk) {
        P.chunks.push_back(make_int4(L.nnodes, s, std::min(e, s + kChunk), 0));
        ++L.nch;
      }
      if (e - a < kCovMinNode) L.cov = false;
      const int c0 = L.ncch;
      for (int s = a; s < e; s += kCovChunk) {
        P.cchunks.push_back(make_int4(L.nnodes, s, std::min(e, s + kCovChunk), 0));
        ++L.ncch;
      }
      P.cnodes.push_back(make_int4(c0, L.ncch, 0, 0));
      ++L.nnodes;
      next.push_back({lo, mid});
      next.push_back({mid, hi});
    }
    if (L.nnodes > 0) {
      P.nodes.push_back(make_int4(0, 0, 0, L.nch));        // sentinel: chunk end of the last node
      P.levels.push_back(L);
      P.max_nodes = std::max(P.max_nodes, L.nnodes);
      P.max_chunks = std::max(P.max_chunks, L.nch);
      if (L.cov) P.max_cchunks = std::max(P.max_cchunks, L.ncch);
    }
    frontier.swap(next);
  }
  return P;
}

}  // namespace

size_t reblock_levels(int N, int block) { return make_plan(N, block).levels.size(); }

ReblockLayout reblock_layout(int H, int N, int d, int block) {
  ReblockLayout L{};
  const Plan P = make_plan(N, block);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) / 256 * 256;
    return at;
  };
  const size_t dd = static_cast<size_t>(d) * d;
  L.mpart = take(static_cast<size_t>(H) * kMomentParts * dd * 4);
  L.M = take(static_cast<size_t>(H) * dd * 4);
  L.W = take(static_cast<size_t>(H) * dd * 4);
  L.Wb = take(static_cast<size_t>(H) * dd * 2);
  L.X = take(static_cast<size_t>(H) * N * d * 2);
  L.perm0 = take(static_cast<size_t>(H) * N * 4);
  L.perm1 = take(static_cast<size_t>(H) * N * 4);
  L.keys = take(static_cast<size_t>(H) * N * 4);
  L.meta = take((P.nodes.size() + P.chunks.size() + P.cnodes.size() + P.cchunks.size()) *
                sizeof(int4));
  const size_t mn = std::max(P.max_nodes, 1), mc = std::max(P.max_chunks, 1);
  L.part = take(static_cast<size_t>(H) * mc * 2 * d * 4);
  L.cpart = take(d == 128 ? static_cast<size_t>(H) * std::max(P.max_cchunks, 1) * kCovStride * 4
                          : 256);
  L.mu = take(static_cast<size_t>(H) * mn * d * 4);
  L.v = take(static_cast<size_t>(H) * mn * d * 4);
  L.hist = take(static_cast<size_t>(H) * mn * 256 * 4);
  L.state = take(static_cast<size_t>(H) * mn * 2 * 4);
  L.cnt = take(static_cast<size_t>(H) * mc * 2 * 4);
  L.base = take(static_cast<size_t>(H) * mc * 3 * 4);
  L.err = take(4);
  L.total = off;
  L.levels = static_cast<int>(P.levels.size());
  L.nb = P.nb;
  return L;
}

constexpr int kMomentTcParts = 6;     // token-tile partitions per head on the tensor cores
constexpr int kWhitenTcTiles = 16;    // token tiles per CTA of the tensor-core whitening

template <int D, typename T>
static cudaError_t whiten_t(const void* Xin, const void* Yin, int H, int N, uint8_t* ws,
                           const ReblockLayout& L, cudaStream_t s) {
  float* part = reinterpret_cast<float*>(ws + L.mpart);
  float* M = reinterpret_cast<float*>(ws + L.M);
  float* W = reinterpret_cast<float*>(ws + L.W);
  auto* Wb = reinterpret_cast<__nv_bfloat16*>(ws + L.Wb);
  auto* X = reinterpret_cast<__nv_bfloat16*>(ws + L.X);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + L.err);
  constexpr bool kTc = (D == 128) && std::is_same<T, __nv_bfloat16>::value;
  const int tiles = (N + 127) / 128;
  CUtensorMap map_x, map_y, map_w;
  if constexpr (kTc) {
    if (!encode_rows_map(&map_x, Xin, H, N, D) || !encode_rows_map(&map_y, Yin, H, N, D) ||
        !encode_rows_map(&map_w, Wb, H, D, D))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaMemsetAsync(err, 0, 4, s);
  if (e != cudaSuccess) return e;
  if constexpr (kTc) {
    const size_t smem = 1024 + kMomStages * kTcTile + 2 * kMomStages * 8 + 8 + 16;
    e = cudaFuncSetAttribute(rb_moment_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    rb_moment_tc_kernel<<<dim3(kMomentTcParts, H), 128, smem, s>>>(map_y, tiles, part, err, wait_limit_ns());
    rb_moment_reduce_kernel<D><<<H, kRbThreads, 0, s>>>(part, kMomentTcParts, N, M);
  } else {
    rb_moment_partial_kernel<D, T><<<dim3(kMomentParts, H), kRbThreads, 0, s>>>(
        static_cast<const T*>(Yin), N, part);
    rb_moment_reduce_kernel<D><<<H, kRbThreads, 0, s>>>(part, kMomentParts, N, M);
  }
  const size_t sq_smem = 3 * D * D * sizeof(float);
  e = cudaFuncSetAttribute(rb_sqrt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sq_smem));
  if (e != cudaSuccess) return e;
  rb_sqrt_kernel<D><<<H, 512, sq_smem, s>>>(M, W, Wb);
  if constexpr (kTc) {
    const size_t smem = 1024 + 3 * kTcTile + 11 * 8 + 16;
    e = cudaFuncSetAttribute(rb_whiten_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int ctas = (tiles + kWhitenTcTiles - 1) / kWhitenTcTiles;
    rb_whiten_tc_kernel<<<dim3(ctas, H), 160, smem, s>>>(map_x, map_w, N, tiles, X, err, wait_limit_ns());
  } else {
    const size_t wh_smem = (D * D + kRbWarps * 8 * D) * sizeof(float);
    e = cudaFuncSetAttribute(rb_whiten_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(wh_smem));
    if (e != cudaSuccess) return e;
    const int tok_per_cta = kRbWarps * 8 * 4;
    rb_whiten_kernel<D, T><<<dim3((N + tok_per_cta - 1) / tok_per_cta, H), kRbThreads, wh_smem,
                             s>>>(static_cast<const T*>(Xin), W, N, X);
  }
  return cudaGetLastError();
}

cudaError_t launch_reblock_whiten(const void* Xin, const void* Yin, int dtype, int H, int N,
                                  int d, void* workspace, const ReblockLayout& L,
                                  cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (d == 128)
    return dtype == 0 ? whiten_t<128, __nv_bfloat16>(Xin, Yin, H, N, ws, L, s)
                      : whiten_t<128, float>(Xin, Yin, H, N, ws, L, s);
  return dtype == 0 ? whiten_t<64, __nv_bfloat16>(Xin, Yin, H, N, ws, L, s)
                    : whiten_t<64, float>(Xin, Yin, H, N, ws, L, s);
}

cudaError_t upload_reblock_plan(int N, int block, void* workspace, const ReblockLayout& L,
                                cudaStream_t s) {
  const Plan P = make_plan(N, block);
  std::vector<int4> meta(P.nodes);
  meta.insert(meta.end(), P.chunks.begin(), P.chunks.end());
  meta.insert(meta.end(), P.cnodes.begin(), P.cnodes.end());
  meta.insert(meta.end(), P.cchunks.begin(), P.cchunks.end());
  if (meta.empty()) return cudaSuccess;
  // pageable source: the copy is staged before the call returns
  return cudaMemcpyAsync(static_cast<uint8_t*>(workspace) + L.meta, meta.data(),
                         meta.size() * sizeof(int4), cudaMemcpyHostToDevice, s);
}

template <int D>
static cudaError_t level_t(int H, int N, int block, int level, const int32_t* perm_in,
                           int32_t* perm_out, uint8_t* ws, const ReblockLayout& L,
                           cudaStream_t s) {
  const Plan P = make_plan(N, block);
  const LevelMeta& lm = P.levels[level];
  const int4* meta = reinterpret_cast<const int4*>(ws + L.meta);
  const int4* nodes = meta + lm.node_off;
  const int4* chunks = meta + P.nodes.size() + lm.chunk_off;
  const int nn = lm.nnodes, nc = lm.nch;
  const auto* X = reinterpret_cast<const __nv_bfloat16*>(ws + L.X);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* mu = reinterpret_cast<float*>(ws + L.mu);
  float* v = reinterpret_cast<float*>(ws + L.v);
  auto* keys = reinterpret_cast<uint32_t*>(ws + L.keys);
  auto* hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  auto* state = reinterpret_cast<uint32_t*>(ws + L.state);
  int* cnt = reinterpret_cast<int*>(ws + L.cnt);
  int* base = reinterpret_cast<int*>(ws + L.base);
  const dim3 gc(nc, H), gn(nn, H);
  cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(H) * nn * 256 * 4, s);
  if (e != cudaSuccess) return e;
  if (D == 128 && lm.cov) {
    const int4* cnodes = meta + P.nodes.size() + P.chunks.size() + lm.cnode_off;
    const int4* cchunks = meta + P.nodes.size() + P.chunks.size() + P.cnodes.size() + lm.cchunk_off;
    float* cpart = reinterpret_cast<float*>(ws + L.cpart);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws + L.err);
    const size_t smem = 1024 + 2 * kTcTile + 3 * 8 + 16 + 256 * 4 + 128 * 8 * 4;
    if (lm.ncch == nn) {
      // every node is one chunk: moments and power iterations in one kernel
      e = cudaFuncSetAttribute(rb_cov_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      rb_cov_tc_kernel<true><<<dim3(lm.ncch, H), 128, smem, s>>>(
          X, perm_in, N, cchunks, lm.ncch, cpart, err, wait_limit_ns(), nn, mu, v);
    } else {
      e = cudaFuncSetAttribute(rb_cov_tc_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      rb_cov_tc_kernel<false><<<dim3(lm.ncch, H), 128, smem, s>>>(
          X, perm_in, N, cchunks, lm.ncch, cpart, err, wait_limit_ns(), nn, mu, v);
      const size_t nsmem = 128 * 128 * 4;
      e = cudaFuncSetAttribute(rb_cov_node_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(nsmem));
      if (e != cudaSuccess) return e;
      rb_cov_node_kernel<<<gn, 128, nsmem, s>>>(cpart, lm.ncch, cnodes, nodes, nn, mu, v);
    }
  } else {
    rb_power_kernel<D, true><<<gc, kRbThreads, 0, s>>>(X, perm_in, N, chunks, nc, v, nn, part);
    rb_node_reduce_kernel<D, true><<<gn, D, 0, s>>>(part, nc, nodes, nn, mu, v);
    for (int it = 1; it < kPowerIters; ++it) {
      rb_power_kernel<D, false><<<gc, kRbThreads, 0, s>>>(X, perm_in, N, chunks, nc, v, nn, part);
      rb_node_reduce_kernel<D, false><<<gn, D, 0, s>>>(part, nc, nodes, nn, mu, v);
    }
  }
  rb_project_kernel<D><<<gc, kRbThreads, 0, s>>>(X, perm_in, N, chunks, v, nn, keys, hist);
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (shift < 24)
      rb_hist_kernel<<<gc, kRbThreads, 0, s>>>(keys, N, chunks, state, nn, hist, shift);
    rb_pick_kernel<<<gn, 32, 0, s>>>(hist, nodes, nn, state, shift);
  }
  rb_count_kernel<<<gc, kRbThreads, 0, s>>>(keys, N, chunks, nc, state, nn, cnt);
  rb_scan_kernel<<<gn, 32, 0, s>>>(cnt, nc, nodes, nn, chunks, state, base);
  e = cudaMemcpyAsync(perm_out, perm_in, static_cast<size_t>(H) * N * 4,
                      cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return e;
  rb_scatter_kernel<<<gc, kRbThreads, 0, s>>>(keys, perm_in, N, chunks, nc, nodes, state, nn,
                                              base, perm_out);
  return cudaGetLastError();
}

cudaError_t launch_reblock_level(int H, int N, int d, int block, int level,
                                 const int32_t* perm_in, int32_t* perm_out, void* workspace,
                                 const ReblockLayout& L, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return d == 128 ? level_t<128>(H, N, block, level, perm_in, perm_out, ws, L, s)
                  : level_t<64>(H, N, block, level, perm_in, perm_out, ws, L, s);
}

__global__ void rb_iota_kernel(int32_t* __restrict__ perm, int N, int H) {
  const size_t n = static_cast<size_t>(N) * H;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    perm[i] = static_cast<int32_t>(i % N);
}

__global__ void rb_offsets_kernel(int32_t* __restrict__ offsets, int nb, int N, int block) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= nb; b += gridDim.x * blockDim.x)
    offsets[b] = b >= nb ? N : b * block;
}

cudaError_t launch_reblock_partition(int H, int N, int d, int block, int32_t* perm_out,
                                     void* workspace, const ReblockLayout& L, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* p0 = reinterpret_cast<int32_t*>(ws + L.perm0);
  int32_t* p1 = reinterpret_cast<int32_t*>(ws + L.perm1);
  rb_iota_kernel<<<148 * 4, 256, 0, s>>>(p0, N, H);
  cudaError_t e = upload_reblock_plan(N, block, workspace, L, s);
  if (e != cudaSuccess) return e;
  for (int lv = 0; lv < L.levels; ++lv) {
    e = launch_reblock_level(H, N, d, block, lv, p0, p1, workspace, L, s);
    if (e != cudaSuccess) return e;
    std::swap(p0, p1);
  }
  return cudaMemcpyAsync(perm_out, p0, static_cast<size_t>(H) * N * 4, cudaMemcpyDeviceToDevice,
                         s);
}

cudaError_t launch_reblock_offsets(int32_t* offsets, int nb, int N, int block, cudaStream_t s) {
  rb_offsets_kernel<<<(nb + 256) / 256, 256, 0, s>>>(offsets, nb, N, block);
  return cudaGetLastError();
}

}  // namespace spark
