// Two-branch block-sparse attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Spark-H3 blog, "Spark-Reblock", BSA equations: for query block A the keys are the exact
// rows of every selected key block plus one summary row per unselected block (section
// "Spark-Reweight": weighted summary k~_B, v~_B with logit offset c_B = b_B + log|B|), and
// a single row-wise softmax normalises both branches.
//
// One CTA per (query block A, head h); 11 warps with fixed roles:
//   warps 0-3  softmax of the EVEN key tiles, warps 4-7 softmax of the ODD key tiles; warp w
//              owns TMEM lanes 32*(w%4).. (query rows) and all 128 columns of its tiles.
//              Each parity keeps its own online softmax (running max, running sum and O
//              accumulator in TMEM) over its half of the tiles, so the two warps of an SMSP
//              never wait for each other and drift out of phase: one is in its exponentials
//              while the other waits for data.  The two partial results are merged once in
//              the epilogue (max-shifted sums), which is exact.  Per tile: read the S row from
//              TMEM twice (row max, then exponentials), apply the scale, the column mask or
//              the summary offsets, rescale lazily (the max used for the exponentials only
//              moves when a tile's max exceeds it by more than 8 in log2 units, and only then
//              is the O row rescaled), and write P (bf16) over the S tile it came from.
//   warp 8     TMA producer: the Q tile once, then K tiles (3-stage ring).
//   warp 9     TMA producer of V tiles (2-stage ring).
//   warp 10    MMA issuer (one thread): S(t) = Q K^T (both from shared memory) into TMEM
//              buffer t%2, O_{t%2} += P(t) V(t) (P read from TMEM, V an MN-major shared-memory
//              operand).  Issue order S(0), S(1), PV(0), S(2), PV(1), S(3), ...: MMAs of one
//              thread execute in order, so S(t+2) overwrites the buffer only after PV(t) has
//              consumed P(t), and the commit of S(t+2) also covers PV(t) - the softmax of
//              tile t+2 may rescale O_{t%2} once it sees S(t+2).
//
// Tile list of a CTA: the k selected blocks in ascending order (a 128-row TMA box starting at
// the block's first row; rows past the block are masked), then ceil(nc/128) tiles of the
// head's context tokens (same blog section: context/sink tokens stay exact, outside the Top-K
// budget; rows past nc masked), then ceil(nkb/128) tiles of the summary rows (rows past nkb
// are zero-filled by TMA and masked, selected blocks masked).
//
// TMEM columns (512 allocated, one CTA per SM): S/P buffer 0 [0,128), buffer 1 [128,256),
// O_even [256,256+D), O_odd [384,384+D).
//
// Every wait is bounded (spark_ptx.cuh); on expiry the kernel flags kErrTimeout, stops every
// role, drains the copies and MMAs it issued, frees TMEM and returns.
#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kWarpK = 8, kWarpV = 9, kWarpMma = 10;
constexpr int kThreads = 352;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kMaxSmemBias = 6144;          // summary offsets kept in shared memory (floats)

// Which of a thread's exponential pairs go to the polynomial (FMA pipe) instead of MUFU.
// Measured at 768p (attention ms, A/B in one run): none 77.1, a quarter 78.7, half 83.1 - the
// softmax here is bound by latency and issue slots, not by MUFU throughput, so all pairs take
// ex2.approx.  The polynomial path stays available (and tested) for kernels where it pays.
__device__ __forceinline__ constexpr bool poly_pair(int) { return false; }

struct __align__(8) Barriers {
  uint64_t qfull;
  uint64_t kfull[kKStages], kempty[kKStages], vfull[kVStages], vempty[kVStages];
  uint64_t sfull[2], pready[2], done;
};

__device__ __forceinline__ bool wait_bounded_ignore_abort(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Row range of key tile t, its source and how many of its 128 rows are valid.
enum TileSrc : int { kSrcVideo = 0, kSrcContext = 1, kSrcSummary = 2 };

struct TileInfo {
  int y;          // first row (in Kp/Vp, in the context rows, or in k~/v~)
  int nvalid;     // exact tiles: valid rows (rows >= nvalid are masked)
  int src;        // TileSrc
  bool exact;     // video or context rows (no summary offset)
};

// Tiles 0..k-1: selected video blocks; then nxt context tiles; then the summary tiles.
__device__ __forceinline__ TileInfo tile_info(int t, int k, int nxt, int nc,
                                              const int32_t* sel_row, const int32_t* k_offsets,
                                              int nkb, int N) {
  TileInfo ti;
  if (t < k) {
    const int B = min(max(sel_row[t], 0), nkb - 1);
    const int lo = min(max(k_offsets[B], 0), N - 1);
    const int hi = min(max(k_offsets[B + 1], lo), N);
    ti.y = lo;
    ti.nvalid = min(hi - lo, kMaxBlock);
    ti.src = kSrcVideo;
    ti.exact = true;
  } else if (t < k + nxt) {
    ti.y = (t - k) * 128;
    ti.nvalid = min(nc - ti.y, 128);
    ti.src = kSrcContext;
    ti.exact = true;
  } else {
    ti.y = (t - k - nxt) * 128;
    ti.nvalid = 128;
    ti.src = kSrcSummary;
    ti.exact = false;
  }
  return ti;
}

// Reads 64 columns of this thread's S row (TMEM) and turns them into logits: exact tiles give
// raw scores (the scale is applied in the exponent) with columns past the block set to -inf;
// summary tiles give s*scale_log2 + offset (offset -inf for selected blocks and padding).
template <bool kBiasSmem>
__device__ __forceinline__ void load_logits(uint32_t taddr, int col0, const TileInfo& ti,
                                            float scale_log2, const float* biasrow,
                                            const float* cb, const uint32_t* selmask, int nkb,
                                            float (&x)[64]) {
  uint32_t r[64];
  tmem_ld64(taddr, r);
#pragma unroll
  for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(r[j]);
  if (ti.exact) {
    if (ti.nvalid < col0 + 64) {
#pragma unroll
      for (int j = 0; j < 64; ++j)
        if (col0 + j >= ti.nvalid) x[j] = -INFINITY;
    }
  } else if (kBiasSmem) {
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
      const float c = cb[Bc];                         // unconditional: the loads batch up
      const uint32_t bits = selmask[Bc >> 5];
      const bool live = B < nkb && !((bits >> (Bc & 31)) & 1u);
      x[j] = live ? fmaf(x[j], scale_log2, c * kLog2e) : -INFINITY;
    }
  }
}

__device__ __forceinline__ float max64(const float (&x)[64]) {
  float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
  for (int j = 4; j < 64; j += 8) {
    mx[0] = fmax3(mx[0], x[j], x[j + 1]);
    mx[1] = fmax3(mx[1], x[j + 2], x[j + 3]);
    mx[2] = fmax3(mx[2], x[j + 4], x[j + 5]);
    mx[3] = fmax3(mx[3], x[j + 6], x[j + 7]);
  }
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
}

// p = 2^(x*c - m) for 64 columns, packed to bf16 pairs; returns the sum of the p.
__device__ __forceinline__ float exp64(const float (&x)[64], float c, float m,
                                       uint32_t (&pk)[32]) {
  const uint64_t c2 = f2_splat(c);
  const uint64_t nm2 = f2_splat(-m);
  uint64_t sum2[4] = {0, 0, 0, 0};
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
  return s0 + s1;
}

}  // namespace

template <int D, bool kBiasSmem>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kt,
    const __grid_constant__ CUtensorMap map_vt, const __grid_constant__ CUtensorMap map_kc,
    const __grid_constant__ CUtensorMap map_vc, int nc, const float* __restrict__ cbias,
    const int32_t* __restrict__ sel, int k, const int32_t* __restrict__ q_perm,
    const int32_t* __restrict__ q_offsets, int nqb, const int32_t* __restrict__ k_offsets,
    int nkb, int N, void* __restrict__ out, int out_dtype, uint32_t* err) {
  constexpr int TILE_BYTES = 128 * D * 2;        // one Q, K or V tile (bf16)
  constexpr int NATOM = D / 64;                  // 128-byte swizzle atoms across d
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qst = smem;
  uint8_t* kst = qst + TILE_BYTES;
  uint8_t* vst = kst + kKStages * TILE_BYTES;
  Barriers* bars = reinterpret_cast<Barriers*>(vst + kVStages * TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* selmask = reinterpret_cast<uint32_t*>(tmem_slot + 4);
  // summary-row offsets of this CTA in log2 units, -inf for selected blocks and padding
  // (16-byte aligned explicitly: the softmax reads it with float4 loads)
  float* biasrow = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(selmask + (nkb + 31) / 32) + 15) & ~static_cast<uintptr_t>(15));

  const int A = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  __shared__ int s_skip;
  __shared__ float ex_m[2][128], ex_l[2][128];   // [parity][row] for the epilogue merge
  if (tid == 0) s_skip = launch_timed_out(err) ? 1 : 0;   // an earlier CTA gave up
  __syncthreads();
  if (s_skip) return;                                      // uniform: no work, nothing held
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  const int nxt = (nc + 127) / 128;                 // context tiles
  const int T = k + nxt + nct;
  const int32_t* sel_row = sel + (static_cast<size_t>(h) * nqb + A) * k;
  const int nwords = (nkb + 31) / 32;
  const float* cb = cbias + static_cast<size_t>(h) * nkb;
  const int qlo = q_offsets[A];

  if (tid == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->sfull[b], 1);
      mbar_init(&bars->pready[b], 4 * 32);
    }
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int i = tid; i < nwords; i += kThreads) selmask[i] = 0u;
  if (kBiasSmem)
    for (int i = tid; i < nct * 128; i += kThreads)
      biasrow[i] = (i < nkb) ? cb[i] * kLog2e : -INFINITY;
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
      if (kBiasSmem) biasrow[B] = -INFINITY;
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
      const int stages = is_k ? kKStages : kVStages;
      uint8_t* ring = is_k ? kst : vst;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      uint64_t* empty = is_k ? bars->kempty : bars->vempty;
      const CUtensorMap* mx = is_k ? &map_k : &map_v;
      const CUtensorMap* mc = is_k ? &map_kc : &map_vc;
      const CUtensorMap* ms = is_k ? &map_kt : &map_vt;
      tma_prefetch_desc(mx);
      tma_prefetch_desc(ms);
      if (nxt > 0) tma_prefetch_desc(mc);
      if (is_k) {
        tma_prefetch_desc(&map_q);
        mbar_arrive_expect_tx(&bars->qfull, TILE_BYTES);
        const int qrow = min(max(qlo, 0), N - 1);   // rows past the block are never stored
        for (int a = 0; a < NATOM; ++a)
          tma_load_3d(qst + a * 16384, &map_q, &bars->qfull, a * 64, qrow, h);
      }
      int issued = 0;
      TileInfo next = tile_info(0, k, nxt, nc, sel_row, k_offsets, nkb, N);
      for (int t = 0; t < T; ++t) {
        const int s = t % stages;
        const TileInfo ti = next;
        if (t >= stages && !mbar_wait(&empty[s], ((t / stages) - 1) & 1, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full[s], TILE_BYTES);
        const CUtensorMap* map = ti.src == kSrcVideo ? mx : (ti.src == kSrcContext ? mc : ms);
        for (int a = 0; a < NATOM; ++a)
          tma_load_3d(ring + s * TILE_BYTES + a * 16384, map, &full[s], a * 64, ti.y, h);
        issued = t + 1;
        if (t + 1 < T) next = tile_info(t + 1, k, nxt, nc, sel_row, k_offsets, nkb, N);
      }
      if (*abort_flag) {
        // drain: wait for every load still in flight (the last round of each stage)
        for (int t = max(0, issued - stages); t < issued; ++t)
          wait_bounded_ignore_abort(&full[t % stages], (t / stages) & 1);
        if (is_k) wait_bounded_ignore_abort(&bars->qfull, 0);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      // descriptors built once; per MMA only a compile-time offset (16-byte units) changes
      const uint64_t qd = sdesc_sw128(smem_u32(qst), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(kst), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(vst), 16384, 1024);
      bool ok = mbar_wait(&bars->qfull, 0, abort_flag, err);
      auto issue_s = [&](int t) -> bool {
        const int s = t % kKStages;
        if (!mbar_wait(&bars->kfull[s], (t / kKStages) & 1, abort_flag, err)) return false;
        const uint32_t dcol = tbase + ((t & 1) ? kColS1 : kColS0);
        const uint64_t kd = kdesc0 + static_cast<uint64_t>(s * (TILE_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * 16384 + (kk % 4) * 32) / 16;
          mma_ss(dcol, qd + off, kd + off, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars->sfull[t & 1]);
        tc_commit(&bars->kempty[s]);
        return true;
      };
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        if (!mbar_wait(&bars->pready[t & 1], (t >> 1) & 1, abort_flag, err)) break;
        tc_fence_after_sync();
        const int s = t % kVStages;
        if (!mbar_wait(&bars->vfull[s], (t / kVStages) & 1, abort_flag, err)) break;
        const uint64_t vd = vdesc0 + static_cast<uint64_t>(s * (TILE_BYTES >> 4));
        const uint32_t pcol = tbase + ((t & 1) ? kColS1 : kColS0);   // P(t) over S(t)
        const uint32_t ocol = tbase + ((t & 1) ? kColO1 : kColO0);
        const uint32_t acc0 = t >= 2 ? 1u : 0u;                       // first tile of a parity
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(ocol, pcol + kk * 8, vd + (kk * 2048) / 16, idO, kk > 0 ? 1u : acc0);
        tc_commit(&bars->vempty[s]);
        if (t + 2 < T && !(ok = issue_s(t + 2))) break;
      }
      // every MMA complete: the softmax epilogue reads O, and TMEM is freed afterwards
      tc_commit(&bars->done);
      wait_bounded_ignore_abort(&bars->done, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax rows
    const int q4 = warp & 3, par = warp >> 2;            // row quarter, tile parity
    const int row = q4 * 32 + lane;                      // 0..127 == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t sbuf = tbase + lane_off + (par ? kColS1 : kColS0);
    const uint32_t obuf = tbase + lane_off + (par ? kColO1 : kColO0);
    const float scale_log2 = kLog2e * rsqrtf(static_cast<float>(D));
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true, first = true;
    TileInfo next = tile_info(par, k, nxt, nc, sel_row, k_offsets, nkb, N);
    for (int t = par; t < T; t += 2) {
      const TileInfo ti = next;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->sfull[par], (t >> 1) & 1, abort_flag, err));
      if (!ok) break;
      tc_fence_after_sync();
      if (t + 2 < T) next = tile_info(t + 2, k, nxt, nc, sel_row, k_offsets, nkb, N);
      const float c = ti.exact ? scale_log2 : 1.f;
      // pass 1: the tile's row maximum (log2 units)
      float x[64];
      load_logits<kBiasSmem>(sbuf, 0, ti, scale_log2, biasrow, cb, selmask, nkb, x);
      float mt = max64(x);
      load_logits<kBiasSmem>(sbuf + 64, 64, ti, scale_log2, biasrow, cb, selmask, nkb, x);
      mt = fmaxf(mt, max64(x));
      if (ti.exact) mt *= scale_log2;                    // -inf stays -inf
      bool need = false;
      float m_new = m_run;
      if (first) {
        m_new = mt;
      } else if (mt > m_run + kRescaleThreshold) {
        need = true;
        m_new = mt;
      }
      // O of this parity is settled (the commit of S(t) covers PV(t-2)); rescale it if the
      // max moved
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2_approx(m_run - m_new) : 1.f;
        l_run *= alpha;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(obuf + cc * 32, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          tmem_st32(obuf + cc * 32, r);
        }
      }
      // pass 2: exponentials, P written over the S columns already consumed
      uint32_t pk[32];
      load_logits<kBiasSmem>(sbuf, 0, ti, scale_log2, biasrow, cb, selmask, nkb, x);
      float rowsum = exp64(x, c, m_new, pk);
      tmem_st32(sbuf, pk);
      load_logits<kBiasSmem>(sbuf + 64, 64, ti, scale_log2, biasrow, cb, selmask, nkb, x);
      rowsum += exp64(x, c, m_new, pk);
      tmem_st32(sbuf + 32, pk);
      l_run = first ? rowsum : l_run + rowsum;
      m_run = m_new;
      first = false;
      tc_fence_before_sync();
      mbar_arrive(&bars->pready[par]);
    }
    // ---- epilogue: merge the two parities and scatter O / l to the original token order
    bool fine = ok && T > 0;
    if (fine) fine = __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, abort_flag, err));
    ex_m[par][row] = m_run;
    ex_l[par][row] = l_run;
    named_bar_sync(1 + q4, 64);                          // the two parities of this quarter
    if (fine) {
      tc_fence_after_sync();
      const float m_o = ex_m[par ^ 1][row], l_o = ex_l[par ^ 1][row];
      const float M = fmaxf(m_run, m_o);
      // weights of the two partial results (a parity without tiles has l = 0)
      const float w_self = l_run > 0.f ? ex2_approx(m_run - M) : 0.f;
      const float w_oth = l_o > 0.f ? ex2_approx(m_o - M) : 0.f;
      const float inv = 1.f / (l_run * w_self + l_o * w_oth);
      const float ws = w_self * inv, wo = w_oth * inv;
      const int qsize = max(0, min(q_offsets[A + 1] - qlo, kMaxBlock));
      int tok = -1;
      if (row < qsize) {
        tok = q_perm[static_cast<size_t>(h) * N + qlo + row];
        if (tok < 0 || tok >= N) {
          if (par == 0) flag_error(err, kErrPerm);
          tok = -1;
        }
      }
      // each parity's warp writes half of the d output columns
      const uint32_t o_self = tbase + lane_off + (par ? kColO1 : kColO0);
      const uint32_t o_oth = tbase + lane_off + (par ? kColO0 : kColO1);
      constexpr int HALF = D / 2;
      // TMEM of a parity that never ran holds garbage: skip it (the weights are 0 there)
      const bool self_live = __any_sync(0xffffffffu, l_run > 0.f);
      const bool oth_live = __any_sync(0xffffffffu, l_o > 0.f);
#pragma unroll
      for (int cc = 0; cc < HALF / 32; ++cc) {
        const int col = par * HALF + cc * 32;
        uint32_t a[32], b[32];
        if (self_live) tmem_ld32(o_self + col, a);
        else for (int j = 0; j < 32; ++j) a[j] = 0u;
        if (oth_live) tmem_ld32(o_oth + col, b);
        else for (int j = 0; j < 32; ++j) b[j] = 0u;
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float av = w_self > 0.f ? __uint_as_float(a[j]) * ws : 0.f;
          const float bv = w_oth > 0.f ? __uint_as_float(b[j]) * wo : 0.f;
          o[j] = av + bv;
        }
        if (tok >= 0) {
          const size_t off = (static_cast<size_t>(h) * N + tok) * D + col;
          if (out_dtype == 0) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + off);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16(o[8 * j], o[8 * j + 1]),
                                  pack_bf16(o[8 * j + 2], o[8 * j + 3]),
                                  pack_bf16(o[8 * j + 4], o[8 * j + 5]),
                                  pack_bf16(o[8 * j + 6], o[8 * j + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
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

static bool bias_in_smem(int nkb, int k) {
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  return nct > 0 && nct * 128 <= kMaxSmemBias;
}

static size_t attend_smem_bytes(int d, int nkb, int k) {
  const size_t tile = static_cast<size_t>(128) * d * 2;
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  const size_t words = (nkb + 31) / 32 + 4;          // + 16 bytes of alignment slack
  const size_t bias = bias_in_smem(nkb, k) ? static_cast<size_t>(nct) * 128 * 4 : 0;
  return 1024 + (1 + kKStages + kVStages) * tile + sizeof(Barriers) + 16 + words * 4 + bias;
}

template <int D, bool kBiasSmem>
static cudaError_t launch_attend_t(const AttendMaps& m, int nc, const float* cbias,
                                   const int32_t* sel, int k, const int32_t* q_perm,
                                   const int32_t* q_offsets,
                                   int nqb, const int32_t* k_offsets, int nkb, int H, int N,
                                   void* out, int out_dtype, uint32_t* err, cudaStream_t s) {
  const size_t smem = attend_smem_bytes(D, nkb, k);
  cudaError_t e = cudaFuncSetAttribute(attend_kernel<D, kBiasSmem>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(nqb, H);
  attend_kernel<D, kBiasSmem><<<grid, kThreads, smem, s>>>(
      m.q, m.k, m.v, m.kt, m.vt, m.kc, m.vc, nc, cbias, sel, k, q_perm, q_offsets, nqb,
      k_offsets, nkb, N, out, out_dtype, err);
  return cudaGetLastError();
}

cudaError_t launch_attend(const AttendMaps& maps, int nc, const float* cbias,
                          const int32_t* sel, int k, const int32_t* q_perm,
                          const int32_t* q_offsets, int nqb, const int32_t* k_offsets, int nkb,
                          int H, int N, int d, void* out, int out_dtype, uint32_t* err,
                          cudaStream_t s) {
  const bool bs = bias_in_smem(nkb, k);
  if (d == 128)
    return bs ? launch_attend_t<128, true>(maps, nc, cbias, sel, k, q_perm, q_offsets, nqb,
                                           k_offsets, nkb, H, N, out, out_dtype, err, s)
              : launch_attend_t<128, false>(maps, nc, cbias, sel, k, q_perm, q_offsets, nqb,
                                            k_offsets, nkb, H, N, out, out_dtype, err, s);
  return bs ? launch_attend_t<64, true>(maps, nc, cbias, sel, k, q_perm, q_offsets, nqb,
                                        k_offsets, nkb, H, N, out, out_dtype, err, s)
            : launch_attend_t<64, false>(maps, nc, cbias, sel, k, q_perm, q_offsets, nqb,
                                         k_offsets, nkb, H, N, out, out_dtype, err, s);
}

}  // namespace spark
