// Two-branch block-sparse attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Spark-H3 blog, "Spark-Reblock", BSA equations: for query block A the keys are the exact
// rows of every selected key block plus one summary row per unselected block (section
// "Spark-Reweight": weighted summary k~_B, v~_B with logit offset c_B = b_B + log|B|), and
// a single row-wise softmax normalises both branches.
//
// One CTA per (query block A, head h); 7 warps with fixed roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  Loads its Q row into TMEM,
//              then per key tile reads the S row from TMEM, applies the scale, the column
//              mask / summary offsets, and an online softmax with lazy rescaling (the running
//              max used for the exponentials only moves when a tile's max exceeds it by more
//              than 8 in log2 units, and only then is the O row in TMEM rescaled); writes P
//              (bf16) into TMEM; finally normalises O and scatters the rows to
//              out[h, q_perm[h, i], :].
//   warp 4     TMA producer of K tiles (3-stage ring).
//   warp 5     TMA producer of V tiles (3-stage ring).
//   warp 6     MMA issuer (one thread): S = Q K^T with Q read from TMEM, O += P V with P read
//              from TMEM; S is double-buffered in TMEM so S(t+2) overlaps softmax(t+1).
//
// Tile list of a CTA: the k selected blocks in ascending order (a 128-row TMA box starting at
// the block's first row; rows past the block are masked), then ceil(nkb/128) tiles of the
// summary rows (rows past nkb are zero-filled by TMA and masked, selected blocks masked).
//
// TMEM columns (512 allocated, one CTA per SM): Q [0,D/2), P [64,128), S0 [128,256),
// S1 [256,384), O [384,384+D).
//
// Every wait is bounded (spark_ptx.cuh); on expiry the kernel flags kErrTimeout, stops every
// role, drains the copies and MMAs it issued, frees TMEM and returns.
#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kStages = 3;
constexpr int kSoftmaxThreads = 256;            // 8 warps: 4 row quarters x 2 column halves
constexpr int kWarpK = 8, kWarpV = 9, kWarpMma = 10;
constexpr int kThreads = 352;
constexpr uint32_t kColQ = 0, kColP = 64, kColS0 = 128, kColS1 = 256, kColO = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kMaxSmemBias = 6144;          // summary offsets kept in shared memory (floats)

// Which of a thread's 32 exponential pairs per tile go to the polynomial (FMA pipe) instead
// of MUFU: 8 of 32, which balances the two pipes against the tensor-core time of a tile.
__device__ __forceinline__ constexpr bool poly_pair(int j) { return (j & 3) == 3; }

struct __align__(8) Barriers {
  uint64_t kfull[kStages], kempty[kStages], vfull[kStages], vempty[kStages];
  uint64_t qready, sfull[2], sfree[2], pready, pvdone, drain;
};

__device__ __forceinline__ bool wait_bounded_ignore_abort(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Row range of key tile t and how many of its 128 rows are valid.
struct TileInfo {
  int y;          // first row (in Kp/Vp for exact tiles, in k~/v~ for summary tiles)
  int nvalid;     // exact tiles: block size (rows >= nvalid are masked)
  bool exact;
};

// Walks the tile list with the metadata of tile t+1 (and the selected id of tile t+2)
// loaded one step ahead, so that the dependent global loads (selected id, then the block's
// offsets) never sit on a role's critical path.
struct TileCursor {
  const int32_t* sel_row;
  const int32_t* k_offsets;
  int k, nkb, N;
  int b_ahead;        // selected id of tile t+2
  TileInfo next;      // metadata of tile t+1

  __device__ __forceinline__ TileInfo info(int t, int B) const {
    TileInfo ti;
    if (t < k) {
      B = min(max(B, 0), nkb - 1);
      const int lo = min(max(k_offsets[B], 0), N - 1);
      const int hi = min(max(k_offsets[B + 1], lo), N);
      ti.y = lo;
      ti.nvalid = min(hi - lo, kMaxBlock);
      ti.exact = true;
    } else {
      ti.y = (t - k) * 128;
      ti.nvalid = 128;
      ti.exact = false;
    }
    return ti;
  }
  __device__ __forceinline__ void init() {
    const int b0 = (k > 0) ? sel_row[0] : 0;
    b_ahead = (k > 1) ? sel_row[1] : 0;
    next = info(0, b0);
  }
  // returns the metadata of tile t and starts the loads for tiles t+1 and t+2
  __device__ __forceinline__ TileInfo advance(int t) {
    const TileInfo cur = next;
    next = info(t + 1, b_ahead);
    b_ahead = (t + 2 < k) ? sel_row[t + 2] : 0;
    return cur;
  }
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(
    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
    const __grid_constant__ CUtensorMap map_kt, const __grid_constant__ CUtensorMap map_vt,
    const __nv_bfloat16* __restrict__ Qp, const float* __restrict__ cbias,
    const int32_t* __restrict__ sel, int k, const int32_t* __restrict__ q_perm,
    const int32_t* __restrict__ q_offsets, int nqb, const int32_t* __restrict__ k_offsets,
    int nkb, int N, void* __restrict__ out, int out_dtype, uint32_t* err) {
  constexpr int TILE_BYTES = 128 * D * 2;        // one K or V tile (bf16)
  constexpr int NATOM = D / 64;                  // 128-byte swizzle atoms across d
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* kst = smem;
  uint8_t* vst = smem + kStages * TILE_BYTES;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + 2 * kStages * TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* selmask = reinterpret_cast<uint32_t*>(tmem_slot + 4);
  // summary-row offsets of this CTA in log2 units, -inf for selected blocks and padding
  // (when nct*128 <= kMaxSmemBias; larger problems read them from global memory)
  float* biasrow = reinterpret_cast<float*>(selmask + ((nkb + 31) / 32 + 3) / 4 * 4);

  const int A = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  __shared__ int s_skip;
  __shared__ float red_max[2][2][128];     // [tile parity][column half][row]
  __shared__ float red_l[2][128];          // [column half][row]
  if (tid == 0) s_skip = launch_timed_out(err) ? 1 : 0;   // an earlier CTA gave up
  __syncthreads();
  if (s_skip) return;                                      // uniform: no work, nothing held
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  const int T = k + nct;
  const int32_t* sel_row = sel + (static_cast<size_t>(h) * nqb + A) * k;
  const int nwords = (nkb + 31) / 32;
  const bool bias_smem = nct > 0 && nct * 128 <= kMaxSmemBias;
  const float* cb = cbias + static_cast<size_t>(h) * nkb;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    mbar_init(&bars->qready, kSoftmaxThreads);
    mbar_init(&bars->sfull[0], 1);
    mbar_init(&bars->sfull[1], 1);
    mbar_init(&bars->pready, kSoftmaxThreads);
    mbar_init(&bars->pvdone, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->sfree[0], kSoftmaxThreads);
    mbar_init(&bars->sfree[1], kSoftmaxThreads);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int i = tid; i < nwords; i += kThreads) selmask[i] = 0u;
  if (bias_smem)
    for (int i = tid; i < nct * 128; i += kThreads) biasrow[i] = (i < nkb) ? cb[i] * kLog2e : -INFINITY;
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  for (int i = tid; i < k; i += kThreads) {
    const int B = sel_row[i];
    if (B >= 0 && B < nkb) {
      atomicOr(&selmask[B >> 5], 1u << (B & 31));
      if (bias_smem) biasrow[B] = -INFINITY;
    } else {
      flag_error(err, kErrSel);
    }
  }
  __syncthreads();
  const uint32_t tbase = *tmem_slot;

  if (warp == kWarpK || warp == kWarpV) {
    // ------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const bool is_k = (warp == kWarpK);
      uint8_t* ring = is_k ? kst : vst;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      const CUtensorMap* mx = is_k ? &map_k : &map_v;
      const CUtensorMap* ms = is_k ? &map_kt : &map_vt;
      tma_prefetch_desc(mx);
      tma_prefetch_desc(ms);
      int issued = 0;
      TileCursor cur{sel_row, k_offsets, k, nkb, N};
      cur.init();
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        const TileInfo ti = cur.advance(t);
        if (t >= kStages && !mbar_wait(&empty[s], ((t / kStages) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full[s], TILE_BYTES);
        for (int a = 0; a < NATOM; ++a)
          tma_load_3d(ring + s * TILE_BYTES + a * 16384, ti.exact ? mx : ms, &full[s], a * 64,
                      ti.y, h);
        issued = t + 1;
      }
      if (*abort_flag) {
        // drain: wait for every load still in flight (the last round of each stage)
        for (int t = max(0, issued - kStages); t < issued; ++t)
          wait_bounded_ignore_abort(&full[t % kStages], (t / kStages) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      bool ok = mbar_wait(&bars->qready, 0, abort_flag, err);
      tc_fence_after_sync();
      auto issue_s = [&](int t) -> bool {
        const int s = t % kStages;
        if (!mbar_wait(&bars->kfull[s], (t / kStages) & 1, abort_flag, err)) return false;
        const uint32_t dcol = tbase + ((t & 1) ? kColS1 : kColS0);
        const uint32_t kaddr = smem_u32(kst + s * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(kaddr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          mma_ts(dcol, tbase + kColQ + kk * 8, bdesc, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars->sfull[t & 1]);
        tc_commit(&bars->kempty[s]);
        return true;
      };
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        // S(t+2) goes into the buffer of S(t) as soon as the softmax has read S(t), so that
        // the tensor cores compute it while the softmax of tile t runs
        if (t + 2 < T) {
          if (!mbar_wait(&bars->sfree[t & 1], (t >> 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after_sync();
          if (!(ok = issue_s(t + 2))) break;
        }
        if (!mbar_wait(&bars->pready, t & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after_sync();
        const int s = t % kStages;
        if (!mbar_wait(&bars->vfull[s], (t / kStages) & 1, abort_flag, err)) { ok = false; break; }
        const uint32_t vaddr = smem_u32(vst + s * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vaddr + kk * 2048, 16384, 1024);
          mma_ts(tbase + kColO, tbase + kColP + kk * 8, bdesc, idO, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars->pvdone);
        tc_commit(&bars->vempty[s]);
      }
      // make sure nothing this thread issued is still running before TMEM is freed
      tc_commit(&bars->drain);
      wait_bounded_ignore_abort(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax rows
    // Warp w handles TMEM lanes 32*(w%4).. (query rows) and S columns 64*(w/4)..+63; the
    // two warps of a row quarter exchange their partial row maxima once per tile.
    const int q4 = warp & 3, half = warp >> 2;
    const int row = q4 * 32 + lane;                       // 0..127 == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t bar_id = 1 + q4;                       // named barrier of the warp pair
    const int col0 = half * 64;                           // first S column of this warp
    constexpr int OH = D / 2;                             // O columns per warp
    const int qlo = q_offsets[A];
    const int qhi = q_offsets[A + 1];
    const int qsize = max(0, min(qhi - qlo, kMaxBlock));
    // this warp's half of the Q row -> TMEM (rows past the block are never stored)
    {
      const int qrow = min(max(qlo, 0), N - 1) + row;
      const bool in = qrow < N;
      const uint32_t* src = reinterpret_cast<const uint32_t*>(
          Qp + (static_cast<size_t>(h) * N + (in ? qrow : 0)) * D) + half * (D / 4);
      if constexpr (D == 128) {
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const uint4 v = in ? *reinterpret_cast<const uint4*>(src + j) : make_uint4(0, 0, 0, 0);
          r[j] = v.x; r[j + 1] = v.y; r[j + 2] = v.z; r[j + 3] = v.w;
        }
        tmem_st32(tbase + lane_off + kColQ + half * 32, r);
      } else {
        uint32_t r[16];
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const uint4 v = in ? *reinterpret_cast<const uint4*>(src + j) : make_uint4(0, 0, 0, 0);
          r[j] = v.x; r[j + 1] = v.y; r[j + 2] = v.z; r[j + 3] = v.w;
        }
        tmem_st16(tbase + lane_off + kColQ + half * 16, r);
      }
    }
    tc_fence_before_sync();
    mbar_arrive(&bars->qready);

    const float scale_log2 = kLog2e * rsqrtf(static_cast<float>(D));
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    TileCursor cur{sel_row, k_offsets, k, nkb, N};
    cur.init();
    // The loop never exits early: the two warps of a row quarter must execute the same
    // sequence of named-barrier exchanges.  After a failed (bounded) wait `ok` stays false
    // for the warp and every later TMEM access, arrival and store of the warp is skipped.
    for (int t = 0; t < T; ++t) {
      const TileInfo ti = cur.advance(t);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->sfull[t & 1], (t >> 1) & 1, abort_flag, err));
      float x[64];
      if (ok) {
        tc_fence_after_sync();
        uint32_t r[64];
        tmem_ld64(tbase + lane_off + ((t & 1) ? kColS1 : kColS0) + col0, r);
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(r[j]);
        // S(t) is in registers: its TMEM buffer may take S(t+2)
        tc_fence_before_sync();
        mbar_arrive(&bars->sfree[t & 1]);
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = -INFINITY;
      }
      // x holds raw scores on exact tiles (scale folded into the exponent below) and
      // log2-domain logits with the summary offsets on summary tiles; masked = -inf.
      if (ti.exact) {
        if (ti.nvalid < col0 + 64) {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (col0 + j >= ti.nvalid) x[j] = -INFINITY;
        }
      } else if (bias_smem) {
        const float4* br = reinterpret_cast<const float4*>(biasrow + ti.y + col0);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float4 b = br[j];
          x[4 * j] = fmaf(x[4 * j], scale_log2, b.x);
          x[4 * j + 1] = fmaf(x[4 * j + 1], scale_log2, b.y);
          x[4 * j + 2] = fmaf(x[4 * j + 2], scale_log2, b.z);
          x[4 * j + 3] = fmaf(x[4 * j + 3], scale_log2, b.w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int B = ti.y + col0 + j;
          const int Bc = min(B, nkb - 1);
          const float c = cb[Bc];                         // unconditional: loads batch up
          const uint32_t bits = selmask[Bc >> 5];
          const bool live = B < nkb && !((bits >> (Bc & 31)) & 1u);
          x[j] = live ? fmaf(x[j], scale_log2, c * kLog2e) : -INFINITY;
        }
      }
      // row maximum of this half: four chains of three-input maxima
      float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int j = 4; j < 64; j += 8) {
        mx[0] = fmax3(mx[0], x[j], x[j + 1]);
        mx[1] = fmax3(mx[1], x[j + 2], x[j + 3]);
        mx[2] = fmax3(mx[2], x[j + 4], x[j + 5]);
        mx[3] = fmax3(mx[3], x[j + 6], x[j + 7]);
      }
      float mloc = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
      if (ti.exact) mloc *= scale_log2;                   // -inf stays -inf
      // combine with the other column half of the same rows (double-buffered slot)
      red_max[t & 1][half][row] = mloc;
      named_bar_sync(bar_id, 64);
      const float mt = fmaxf(mloc, red_max[t & 1][half ^ 1][row]);
      bool need = false;
      float m_new = m_run;
      if (t == 0) {
        m_new = mt;
      } else if (mt > m_run + kRescaleThreshold) {
        need = true;
        m_new = mt;
      }
      // p = 2^(x*c - m) on exact tiles (raw scores), 2^(x - m) on summary tiles, two
      // columns at a time; a quarter of the pairs use the FMA-pipe polynomial
      const uint64_t c2 = f2_splat(ti.exact ? scale_log2 : 1.f);
      const uint64_t nm2 = f2_splat(-m_new);
      uint64_t sum2[4] = {0, 0, 0, 0};
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint64_t a2 = f2_fma(f2_pack(x[2 * j], x[2 * j + 1]), c2, nm2);
        float p0, p1;
        if (poly_pair(j)) {
          exp2_poly2(a2, p0, p1);
        } else {
          float a0, a1;
          f2_unpack(a2, a0, a1);
          p0 = ex2_approx(a0);
          p1 = ex2_approx(a1);
        }
        sum2[j & 3] = f2_add(sum2[j & 3], f2_pack(p0, p1));
        pk[j] = pack_bf16(p0, p1);
      }
      float s0, s1;
      f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
      const float rowsum = s0 + s1;
      // P and O of the previous tile are in use until its PV MMA completes
      if (ok && t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->pvdone, (t - 1) & 1, abort_flag, err));
        if (ok) tc_fence_after_sync();
      }
      if (!ok) continue;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.f;
        l_run *= alpha;
#pragma unroll
        for (int c = 0; c < OH / 32; ++c) {
          uint32_t r[32];
          const uint32_t oa = tbase + lane_off + kColO + half * OH + c * 32;
          tmem_ld32(oa, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          tmem_st32(oa, r);
        }
      }
      l_run += rowsum;
      m_run = m_new;
      tmem_st32(tbase + lane_off + kColP + half * 32, pk);
      tc_fence_before_sync();
      mbar_arrive(&bars->pready);
    }
    // ---- epilogue: O / l scattered to the original token order
    bool fine = ok && T > 0;
    if (fine) fine = mbar_wait(&bars->pvdone, (T - 1) & 1, abort_flag, err);
    fine = __all_sync(0xffffffffu, fine);
    // the pair exchanges its partial row sums (both warps always reach this barrier)
    red_l[half][row] = l_run;
    named_bar_sync(bar_id, 64);
    if (fine) {
      const float l_tot = l_run + red_l[half ^ 1][row];
      tc_fence_after_sync();
      const float inv = 1.f / l_tot;
      int tok = -1;
      if (row < qsize) {
        tok = q_perm[static_cast<size_t>(h) * N + qlo + row];
        if (tok < 0 || tok >= N) {
          if (half == 0) flag_error(err, kErrPerm);
          tok = -1;
        }
      }
#pragma unroll
      for (int c = 0; c < OH / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + lane_off + kColO + half * OH + c * 32, r);
        if (tok >= 0) {
          const size_t o = (static_cast<size_t>(h) * N + tok) * D + half * OH + c * 32;
          if (out_dtype == 0) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(r[8 * j + 0]) * inv, __uint_as_float(r[8 * j + 1]) * inv);
              v.y = pack_bf16(__uint_as_float(r[8 * j + 2]) * inv, __uint_as_float(r[8 * j + 3]) * inv);
              v.z = pack_bf16(__uint_as_float(r[8 * j + 4]) * inv, __uint_as_float(r[8 * j + 5]) * inv);
              v.w = pack_bf16(__uint_as_float(r[8 * j + 6]) * inv, __uint_as_float(r[8 * j + 7]) * inv);
              dst[j] = v;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(__uint_as_float(r[4 * j]) * inv, __uint_as_float(r[4 * j + 1]) * inv,
                                   __uint_as_float(r[4 * j + 2]) * inv, __uint_as_float(r[4 * j + 3]) * inv);
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, 512);
  }
}

static size_t attend_smem_bytes(int d, int nkb, int k) {
  const size_t tile = static_cast<size_t>(128) * d * 2;
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  const size_t words = ((nkb + 31) / 32 + 3) / 4 * 4;
  const size_t bias = (nct > 0 && nct * 128 <= kMaxSmemBias) ? static_cast<size_t>(nct) * 128 * 4 : 0;
  return 1024 + 2 * kStages * tile + sizeof(Barriers) + 16 + words * 4 + bias;
}

template <int D>
static cudaError_t launch_attend_t(const AttendMaps& m, const float* cbias, const int32_t* sel,
                                   int k, const int32_t* q_perm, const int32_t* q_offsets,
                                   int nqb, const int32_t* k_offsets, int nkb, int H, int N,
                                   void* out, int out_dtype, uint32_t* err, cudaStream_t s) {
  const size_t smem = attend_smem_bytes(D, nkb, k);
  cudaError_t e = cudaFuncSetAttribute(attend_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(nqb, H);
  attend_kernel<D><<<grid, kThreads, smem, s>>>(m.k, m.v, m.kt, m.vt,
                                                 static_cast<const __nv_bfloat16*>(m.q_base),
                                                 cbias, sel, k, q_perm, q_offsets, nqb, k_offsets,
                                                 nkb, N, out, out_dtype, err);
  return cudaGetLastError();
}

cudaError_t launch_attend(const AttendMaps& maps, const float* cbias, const int32_t* sel, int k,
                          const int32_t* q_perm, const int32_t* q_offsets, int nqb,
                          const int32_t* k_offsets, int nkb, int H, int N, int d, void* out,
                          int out_dtype, uint32_t* err, cudaStream_t s) {
  if (d == 128)
    return launch_attend_t<128>(maps, cbias, sel, k, q_perm, q_offsets, nqb, k_offsets, nkb, H,
                                N, out, out_dtype, err, s);
  return launch_attend_t<64>(maps, cbias, sel, k, q_perm, q_offsets, nqb, k_offsets, nkb, H, N,
                             out, out_dtype, err, s);
}

}  // namespace spark
