// Gather / block-mean / anchor / summary kernels (HBM-bound steps of the forward pass).
//
//  gather_q_kernel          Qp = bf16(Q[q_perm]) and the query-block means.
//                           Spark-H3 blog, "Spark-Reblock" (token permutation into blocks)
//                           and "Discussion" (blocks scored from block-level means).
//  anchor_kernel            qbar[h] = mean of all N queries of head h, from the block means.
//                           Spark-H3 blog, "Spark-Reweight" (the mean of the video queries is
//                           the representative query); comfyui-wiki article (one anchor per
//                           head).
//  gather_kv_summary_kernel Kp, Vp = bf16(K[k_perm]), bf16(V[k_perm]) fused with the key-block
//                           means and the Spark-Reweight summaries: in-block softmax of the
//                           anchor logits, weighted k~/v~, and c = LSE(s) - sigma qbar.k~
//                           (the log-mass bias plus log|B|).  Spark-H3 blog, "Spark-Reweight".
//
// Layout: one CTA per (block, head), 128 threads; a row of d elements is split into d/8
// chunks of 8 elements (16 bytes of bf16), so 128/(d/8) rows are in flight per CTA step.
// Every permutation entry and block boundary is checked before it is used; bad values set
// bits of the error word and the access is skipped.
#include "spark_kernels.cuh"

namespace spark {

namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Loads 8 consecutive elements and returns them as bf16 (packed) and as the fp32 values of
// those bf16 numbers.  fp32 inputs are rounded to nearest-even bf16.
struct Row8 {
  uint4 packed;
};

__device__ __forceinline__ Row8 load8(const __nv_bfloat16* p) { return Row8{ld_stream_v4(p)}; }

__device__ __forceinline__ Row8 load8(const float* p) {
  const uint4 a = ld_stream_v4(p);
  const uint4 b = ld_stream_v4(p + 4);
  Row8 r;
  r.packed.x = pack_bf16(__uint_as_float(a.x), __uint_as_float(a.y));
  r.packed.y = pack_bf16(__uint_as_float(a.z), __uint_as_float(a.w));
  r.packed.z = pack_bf16(__uint_as_float(b.x), __uint_as_float(b.y));
  r.packed.w = pack_bf16(__uint_as_float(b.z), __uint_as_float(b.w));
  return r;
}

// Block [lo, hi) of the offsets array, validated.
__device__ __forceinline__ bool block_bounds(const int32_t* offsets, int b, int N, int& lo,
                                             int& hi) {
  lo = offsets[b];
  hi = offsets[b + 1];
  return lo >= 0 && hi <= N && hi > lo && hi - lo <= kMaxBlock;
}

}  // namespace

// ------------------------------------------------------------------------------ gather_q

template <int D, typename T>
__global__ void __launch_bounds__(128) gather_q_kernel(const T* __restrict__ Q,
                                                       const int32_t* __restrict__ q_perm,
                                                       const int32_t* __restrict__ q_offsets,
                                                       int N, int nqb,
                                                       __nv_bfloat16* __restrict__ Qp,
                                                       float* __restrict__ qbar_blocks,
                                                       uint32_t* err) {
  constexpr int CPR = D / 8;          // 16-byte chunks per row
  constexpr int RG = 128 / CPR;       // rows in flight per step
  __shared__ float red[RG][D];
  const int A = blockIdx.x, h = blockIdx.y;
  const int c = threadIdx.x % CPR, g = threadIdx.x / CPR;
  int lo, hi;
  if (!block_bounds(q_offsets, A, N, lo, hi)) {
    if (threadIdx.x == 0) flag_error(err, kErrOffsets);
    return;
  }
  const int m = hi - lo;
  const size_t head = static_cast<size_t>(h) * N;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  constexpr int U = 4;
  for (int r0 = g; r0 < m; r0 += RG * U) {
    Row8 v[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG;
      ok[u] = false;
      if (r < m) {
        const int t = q_perm[head + lo + r];
        ok[u] = (t >= 0 && t < N);
        if (ok[u]) v[u] = load8(Q + (head + t) * D + c * 8);
        else flag_error(err, kErrPerm);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG;
      if (r < m) {
        if (!ok[u]) v[u].packed = make_uint4(0, 0, 0, 0);
        st_v4(Qp + (head + lo + r) * D + c * 8, v[u].packed);
        float f[8];
        unpack_bf16x8(v[u].packed, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f[e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[g][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int gg = 0; gg < RG; ++gg) s += red[gg][threadIdx.x];
    qbar_blocks[(static_cast<size_t>(h) * nqb + A) * D + threadIdx.x] = s / static_cast<float>(m);
  }
}

// -------------------------------------------------------------------------------- anchor

// One CTA of 1024 threads per head: 1024/D groups each sum a strided subset of the
// size-weighted block means; the groups are combined in a fixed order.
template <int D>
__global__ void __launch_bounds__(1024) anchor_kernel(const float* __restrict__ qbar_blocks,
                                                      const int32_t* __restrict__ q_offsets,
                                                      int N, int nqb, float* __restrict__ qbar) {
  constexpr int G = 1024 / D;
  __shared__ float red[G][D];
  const int h = blockIdx.x;
  const int col = threadIdx.x % D, g = threadIdx.x / D;
  const float* base = qbar_blocks + static_cast<size_t>(h) * nqb * D + col;
  float s = 0.f;
#pragma unroll 8
  for (int A = g; A < nqb; A += G) {
    const float sz = static_cast<float>(q_offsets[A + 1] - q_offsets[A]);
    s += sz * base[static_cast<size_t>(A) * D];
  }
  red[g][col] = s;
  __syncthreads();
  if (threadIdx.x < D) {
    float t = 0.f;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) t += red[gg][threadIdx.x];
    qbar[static_cast<size_t>(h) * D + threadIdx.x] = t / static_cast<float>(N);
  }
}

// ------------------------------------------------------------------ gather_kv + summaries

// kMeanPool: the baseline BSA compressed branch instead of Spark-Reweight's (blog
// "Spark-Reblock", BSA equations: each unselected block repeats its uniform mean key and value
// |B| times; as one row that is k~ = mean key, v~ = mean value, offset c = log|B|).
template <int D, typename T, bool kMeanPool = false>
__global__ void __launch_bounds__(128) gather_kv_summary_kernel(
    const T* __restrict__ K, const T* __restrict__ V, const int32_t* __restrict__ k_perm,
    const int32_t* __restrict__ k_offsets, int N, int nkb, const float* __restrict__ qbar,
    __nv_bfloat16* __restrict__ Kp, __nv_bfloat16* __restrict__ Vp, float* __restrict__ kbar,
    __nv_bfloat16* __restrict__ k_tilde, __nv_bfloat16* __restrict__ v_tilde,
    float* __restrict__ cbias, uint32_t* err) {
  constexpr int CPR = D / 8;
  constexpr int RG = 128 / CPR;
  __shared__ float s_m[RG], s_l[RG];
  __shared__ float s_k[RG][D], s_v[RG][D], s_ks[RG][D];
  __shared__ float s_dot[4];
  const int B = blockIdx.x, h = blockIdx.y;
  const int c = threadIdx.x % CPR, g = threadIdx.x / CPR;
  const size_t bidx = static_cast<size_t>(h) * nkb + B;
  int lo, hi;
  if (!block_bounds(k_offsets, B, N, lo, hi)) {
    if (threadIdx.x == 0) {
      flag_error(err, kErrOffsets);
      cbias[bidx] = -INFINITY;
    }
    if (threadIdx.x < D) {
      kbar[(static_cast<size_t>(h) * D + threadIdx.x) * nkb + B] = 0.f;   // d-major
      k_tilde[bidx * D + threadIdx.x] = __float2bfloat16_rn(0.f);
      v_tilde[bidx * D + threadIdx.x] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int m = hi - lo;
  const size_t head = static_cast<size_t>(h) * N;
  const float sigma = rsqrtf(static_cast<float>(D));
  float qs[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    qs[e] = kMeanPool ? 0.f : sigma * qbar[static_cast<size_t>(h) * D + c * 8 + e];   // no anchor

  float run_m = -INFINITY, run_l = 0.f;
  float ak[8], av[8], ks[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) ak[e] = av[e] = ks[e] = 0.f;

  // The trip count must be the same for every lane of a warp (the row reduction below is a
  // full-warp shuffle), so the loop runs over row groups and each lane derives its row.
  constexpr int U = 2;
  for (int r0 = 0; r0 < m; r0 += RG * U) {
    Row8 kv[U], vv[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG + g;
      ok[u] = false;
      if (r < m) {
        const int t = k_perm[head + lo + r];
        ok[u] = (t >= 0 && t < N);
        if (ok[u]) {
          kv[u] = load8(K + (head + t) * D + c * 8);
          vv[u] = load8(V + (head + t) * D + c * 8);
        } else {
          flag_error(err, kErrPerm);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG + g;
      const bool live = r < m;      // uniform across the CPR threads of one row
      if (!live || !ok[u]) kv[u].packed = vv[u].packed = make_uint4(0, 0, 0, 0);
      float fk[8], fv[8];
      unpack_bf16x8(kv[u].packed, fk);
      unpack_bf16x8(vv[u].packed, fv);
      if constexpr (kMeanPool) {
        if (live) {
          st_v4(Kp + (head + lo + r) * D + c * 8, kv[u].packed);
          st_v4(Vp + (head + lo + r) * D + c * 8, vv[u].packed);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ks[e] += fk[e];
            av[e] += fv[e];                       // the value sum
          }
        }
        continue;
      }
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qs[e], fk[e], dot);
      // every lane of the warp takes part in the row reduction
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (live) {
        st_v4(Kp + (head + lo + r) * D + c * 8, kv[u].packed);
        st_v4(Vp + (head + lo + r) * D + c * 8, vv[u].packed);
        const float new_m = fmaxf(run_m, dot);
        const float a = expf(run_m - new_m);      // 0 for the first row of this thread
        const float p = expf(dot - new_m);
        run_l = run_l * a + p;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ak[e] = fmaf(p, fk[e], ak[e] * a);
          av[e] = fmaf(p, fv[e], av[e] * a);
          ks[e] += fk[e];
        }
        run_m = new_m;
      }
    }
  }
  if (c == 0) {
    s_m[g] = run_m;
    s_l[g] = run_l;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    s_k[g][c * 8 + e] = ak[e];
    s_v[g][c * 8 + e] = av[e];
    s_ks[g][c * 8 + e] = ks[e];
  }
  __syncthreads();
  if constexpr (kMeanPool) {
    if (threadIdx.x < D) {
      const int col = threadIdx.x;
      float ksum = 0.f, vsum = 0.f;
#pragma unroll
      for (int gg = 0; gg < RG; ++gg) {
        ksum += s_ks[gg][col];
        vsum += s_v[gg][col];
      }
      const float inv_m = 1.f / static_cast<float>(m);
      k_tilde[bidx * D + col] = __float2bfloat16_rn(ksum * inv_m);
      v_tilde[bidx * D + col] = __float2bfloat16_rn(vsum * inv_m);
      kbar[(static_cast<size_t>(h) * D + col) * nkb + B] = ksum / static_cast<float>(m);
      if (col == 0) cbias[bidx] = logf(static_cast<float>(m));
    }
    return;
  }
  if (threadIdx.x < D) {
    const int col = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int gg = 0; gg < RG; ++gg) M = fmaxf(M, s_m[gg]);
    float L = 0.f, kk = 0.f, vv = 0.f, ksum = 0.f;
#pragma unroll
    for (int gg = 0; gg < RG; ++gg) {
      const float w = (s_l[gg] > 0.f) ? expf(s_m[gg] - M) : 0.f;
      L = fmaf(s_l[gg], w, L);
      kk = fmaf(s_k[gg][col], w, kk);
      vv = fmaf(s_v[gg][col], w, vv);
      ksum += s_ks[gg][col];
    }
    const float inv = 1.f / L;
    const __nv_bfloat16 kt = __float2bfloat16_rn(kk * inv);
    k_tilde[bidx * D + col] = kt;
    v_tilde[bidx * D + col] = __float2bfloat16_rn(vv * inv);
    // d-major [H][D][nkb]: the routing kernel reads one coalesced row per dimension
    kbar[(static_cast<size_t>(h) * D + col) * nkb + B] = ksum / static_cast<float>(m);
    // sigma * qbar . bf16(k~), reduced over the D columns (D/32 warps)
    float dq = sigma * qbar[static_cast<size_t>(h) * D + col] * __bfloat162float(kt);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dq += __shfl_xor_sync(0xffffffffu, dq, off);
    if ((col & 31) == 0) s_dot[col >> 5] = dq;
    if (col == 0) s_l[0] = M + logf(L);            // LSE of the anchor logits
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float dot = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) dot += s_dot[w];
    cbias[bidx] = s_l[0] - dot;
  }
}

// ----------------------------------------------------------------------------- launchers

template <int D, typename T>
static cudaError_t launch_gather_q_t(const void* Q, int H, int N, const int32_t* q_perm,
                                     const int32_t* q_offsets, int nqb, void* Qp,
                                     float* qbar_blocks, uint32_t* err, cudaStream_t s) {
  dim3 grid(nqb, H);
  gather_q_kernel<D, T><<<grid, 128, 0, s>>>(static_cast<const T*>(Q), q_perm, q_offsets, N,
                                            nqb, static_cast<__nv_bfloat16*>(Qp), qbar_blocks,
                                            err);
  return cudaGetLastError();
}

cudaError_t launch_gather_q(const void* Q, int dtype, int H, int N, int d,
                            const int32_t* q_perm, const int32_t* q_offsets, int nqb, void* Qp,
                            float* qbar_blocks, uint32_t* err, cudaStream_t s) {
  if (d == 128)
    return dtype == 0 ? launch_gather_q_t<128, __nv_bfloat16>(Q, H, N, q_perm, q_offsets, nqb,
                                                               Qp, qbar_blocks, err, s)
                      : launch_gather_q_t<128, float>(Q, H, N, q_perm, q_offsets, nqb, Qp,
                                                      qbar_blocks, err, s);
  return dtype == 0 ? launch_gather_q_t<64, __nv_bfloat16>(Q, H, N, q_perm, q_offsets, nqb, Qp,
                                                            qbar_blocks, err, s)
                    : launch_gather_q_t<64, float>(Q, H, N, q_perm, q_offsets, nqb, Qp,
                                                   qbar_blocks, err, s);
}

cudaError_t launch_anchor(const float* qbar_blocks, const int32_t* q_offsets, int H, int N,
                          int d, int nqb, float* qbar, cudaStream_t s) {
  if (d == 128) anchor_kernel<128><<<H, 1024, 0, s>>>(qbar_blocks, q_offsets, N, nqb, qbar);
  else anchor_kernel<64><<<H, 1024, 0, s>>>(qbar_blocks, q_offsets, N, nqb, qbar);
  return cudaGetLastError();
}

template <int D, typename T, bool kMeanPool = false>
static cudaError_t launch_kv_t(const void* K, const void* V, int H, int N,
                               const int32_t* k_perm, const int32_t* k_offsets, int nkb,
                               const float* qbar, void* Kp, void* Vp, float* kbar,
                               void* k_tilde, void* v_tilde, float* cbias, uint32_t* err,
                               cudaStream_t s) {
  dim3 grid(nkb, H);
  gather_kv_summary_kernel<D, T, kMeanPool><<<grid, 128, 0, s>>>(
      static_cast<const T*>(K), static_cast<const T*>(V), k_perm, k_offsets, N, nkb, qbar,
      static_cast<__nv_bfloat16*>(Kp), static_cast<__nv_bfloat16*>(Vp), kbar,
      static_cast<__nv_bfloat16*>(k_tilde), static_cast<__nv_bfloat16*>(v_tilde), cbias, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_kv_summary(const void* K, const void* V, int dtype, int H, int N,
                                     int d, const int32_t* k_perm, const int32_t* k_offsets,
                                     int nkb, const float* qbar, void* Kp, void* Vp,
                                     float* kbar, void* k_tilde, void* v_tilde, float* cbias,
                                     uint32_t* err, cudaStream_t s) {
  if (d == 128)
    return dtype == 0
               ? launch_kv_t<128, __nv_bfloat16>(K, V, H, N, k_perm, k_offsets, nkb, qbar, Kp,
                                                 Vp, kbar, k_tilde, v_tilde, cbias, err, s)
               : launch_kv_t<128, float>(K, V, H, N, k_perm, k_offsets, nkb, qbar, Kp, Vp,
                                         kbar, k_tilde, v_tilde, cbias, err, s);
  return dtype == 0
             ? launch_kv_t<64, __nv_bfloat16>(K, V, H, N, k_perm, k_offsets, nkb, qbar, Kp, Vp,
                                              kbar, k_tilde, v_tilde, cbias, err, s)
             : launch_kv_t<64, float>(K, V, H, N, k_perm, k_offsets, nkb, qbar, Kp, Vp, kbar,
                                      k_tilde, v_tilde, cbias, err, s);
}

cudaError_t launch_gather_kv_meanpool(const void* K, const void* V, int dtype, int H, int N,
                                      int d, const int32_t* k_perm, const int32_t* k_offsets,
                                      int nkb, void* Kp, void* Vp, float* kbar, void* k_tilde,
                                      void* v_tilde, float* cbias, uint32_t* err,
                                      cudaStream_t s) {
  if (d == 128)
    return dtype == 0
               ? launch_kv_t<128, __nv_bfloat16, true>(K, V, H, N, k_perm, k_offsets, nkb,
                                                       nullptr, Kp, Vp, kbar, k_tilde, v_tilde,
                                                       cbias, err, s)
               : launch_kv_t<128, float, true>(K, V, H, N, k_perm, k_offsets, nkb, nullptr, Kp,
                                               Vp, kbar, k_tilde, v_tilde, cbias, err, s);
  return dtype == 0
             ? launch_kv_t<64, __nv_bfloat16, true>(K, V, H, N, k_perm, k_offsets, nkb, nullptr,
                                                    Kp, Vp, kbar, k_tilde, v_tilde, cbias, err,
                                                    s)
             : launch_kv_t<64, float, true>(K, V, H, N, k_perm, k_offsets, nkb, nullptr, Kp, Vp,
                                            kbar, k_tilde, v_tilde, cbias, err, s);
}

// Context rows to bf16 (round to nearest even), four elements per thread and iteration.
__global__ void __launch_bounds__(256) to_bf16_kernel(const float4* __restrict__ src, size_t n4,
                                                     uint2* __restrict__ dst) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    dst[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                        *reinterpret_cast<const uint32_t*>(&hi));
  }
}

cudaError_t launch_to_bf16(const void* src, int dtype, size_t n, void* dst, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (dtype == 0) return cudaMemcpyAsync(dst, src, n * 2, cudaMemcpyDeviceToDevice, s);
  const size_t n4 = n / 4;                       // n is a multiple of d (64 or 128)
  const size_t blocks = (n4 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(blocks < 148 * 16 ? blocks : 148 * 16);
  to_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const float4*>(src), n4,
                                      static_cast<uint2*>(dst));
  return cudaGetLastError();
}

}  // namespace spark
