// Two-branch block-sparse attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Spark-H3 blog, "Spark-Reblock", BSA equations: for query block A the keys are the exact
// rows of every selected key block plus one summary row per unselected block (section
// "Spark-Reweight": weighted summary k~_B, v~_B with logit offset c_B = b_B + log|B|), and
// a single row-wise softmax normalises both branches.
//
// One CTA per (query block A, head h); 11 warps with fixed roles:
//   warps 0-3  softmax of the even key tiles, warps 4-7 of the odd key tiles (two groups);
//              warp w owns TMEM lanes 32*(w%4).. (query rows).  Both groups exponentiate
//              against one fixed reference per row, the larger of the two groups' first-tile
//              row maxima, so no tile ever rescales anything: P(t) = 2^(s*scale - ref) is
//              written (bf16) over the S columns it came from, each group sums its p, and the
//              epilogue divides the single O accumulator by the two sums.  The exponentials
//              are those of the exact softmax up to the common factor 2^(max - ref), which
//              cancels in the division, so no accuracy is lost as long as every p stays in
//              floating-point range.  A row whose sum leaves [2^-60, 2^60] (a maximum far above
//              the reference, e.g. a sink or context key 50 nats above the first blocks)
//              makes its CTA repeat all tiles (a second pass over the same pipeline): such
//              rows take their recorded maximum as the reference - each chunk whose sum is out
//              of range records its maximum, which is within a few units of the row's - and the
//              other rows keep theirs.
//   warp 8     TMA producer: the Q tile once, then K tiles (3-stage ring; a stage is free
//              again once the S MMA that read it has completed, signalled by that S buffer's
//              barrier).
//   warp 9     TMA producer of V tiles (2-stage ring).
//   warp 10    MMA issuer: S(t) = Q K^T (both from shared memory) into TMEM buffer t%3,
//              O += P(t) V(t) (P read from TMEM, V an MN-major shared-memory operand).  Issue
//              order S(0), S(1), S(2), PV(0), S(3), PV(1), S(4), ...: MMAs of one thread execute
//              in order, so S(t+3) overwrites its buffer only after PV(t) has consumed P(t).
//              With three buffers the next S of a group is ready while the group still works
//              on its current tile.
//   Warps 8-10 run their loops warp-uniformly (stage indices, coordinates and descriptors are
//   the same in every lane) and one elected lane issues the copies, MMAs and commits: issuing
//   from a single divergent lane measured 8% slower at 768p.
//
// Tile list of a CTA: the k selected blocks in ascending order (a 128-row TMA box starting at
// the block's first row; rows past the block are masked), then ceil(nc/128) tiles of the
// head's context tokens (same blog section: context/sink tokens stay exact, outside the Top-K
// budget; rows past nc masked), then ceil(nkb/128) tiles of the summary rows (rows past nkb
// are zero-filled by TMA and masked, selected blocks masked).  When some key block is shorter
// than 128 rows (kVarTiles), an exact tile's S MMA has N = its rows rounded up to 16, its PV
// takes only that many keys, and the softmax covers only those columns.
//
// With the routing inside (kPersist: Spark-H3 blog, "Related Works", Sol-Attn's single pass
// over routing and attention): one persistent CTA per SM walks the query blocks head-major, and
// a 12th warp scores and selects the NEXT query block (route_step.cuh, the routing kernel's
// arithmetic) into a second set of shared-memory buffers while the current one is attended.
//
// TMEM columns (512 allocated, one CTA per SM): S/P buffers [0,128), [128,256), [256,384),
// O [384,384+D).
//
// Every wait is bounded by the launch parameter wait_ns (the library's process-wide setting,
// 4 s by default); on expiry the kernel flags kErrTimeout, stops every role, drains the copies
// and MMAs it issued (waits bounded by the default limit), frees TMEM and returns.
#include <type_traits>

#include "route_step.cuh"

#include "spark_kernels.cuh"

namespace spark {

namespace {

constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kWarpK = 8, kWarpV = 9, kWarpMma = 10;
constexpr int kWarpRoute = 11;              // with in-kernel routing only
constexpr int kThreads = 352;               // 11 warps
constexpr int kThreadsFused = 384;          // 12 warps: 3 per SM sub-partition, 168 registers each
constexpr uint32_t kColO = 384;             // S/P buffer b at column 128*b (b < 3)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxSmemBias = 6144;          // summary offsets kept in shared memory (floats)

struct __align__(8) Barriers {
  uint64_t qfull;
  // the K ring's stages are released by sfull: K stage and S buffer of a tile coincide
  uint64_t kfull[kKStages], vfull[kVStages], vempty[kVStages];
  uint64_t sfull[3], pready[3], done;
  // keys the MMAs of a tile cover (its valid rows rounded up to 16; 128 for summary tiles):
  // written by the K producer per stage before the stage's loads, read by the MMA thread
  uint32_t kn[kKStages];
  uint32_t bn[3];                              // the MMA thread's copy per S buffer
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
  float ks;       // FP8 keys: the tile's scale (its key block's, or its 128-row tile's); else 1
};

// Scales of the FP8 operands (all null for bf16 operands): per query block [H,nqb], per key
// block [H,nkb], per 128-row tile of the summary rows [H,ceil(nkb/128)] and of the context
// rows [H,ceil(nc/128)].
struct Fp8Scales {
  const float* q;
  const float* k;
  const float* kt;
  const float* kc;
};

// Tiles 0..k-1: selected video blocks; then nxt context tiles; then the summary tiles.
template <bool kFp8>
__device__ __forceinline__ TileInfo tile_info(int t, int k, int nxt, int nc,
                                              const int32_t* sel_row, const int32_t* k_offsets,
                                              int nkb, int N, const Fp8Scales& sc, int h) {
  TileInfo ti;
  ti.ks = 1.f;
  if (t < k) {
    const int B = min(max(sel_row[t], 0), nkb - 1);
    const int lo = min(max(k_offsets[B], 0), N - 1);
    const int hi = min(max(k_offsets[B + 1], lo), N);
    ti.y = lo;
    ti.nvalid = min(hi - lo, kMaxBlock);
    ti.src = kSrcVideo;
    ti.exact = true;
    if (kFp8) ti.ks = sc.k[static_cast<size_t>(h) * nkb + B];
  } else if (t < k + nxt) {
    ti.y = (t - k) * 128;
    ti.nvalid = min(nc - ti.y, 128);
    ti.src = kSrcContext;
    ti.exact = true;
    if (kFp8) ti.ks = sc.kc[static_cast<size_t>(h) * nxt + (t - k)];
  } else {
    ti.y = (t - k - nxt) * 128;
    ti.nvalid = 128;
    ti.src = kSrcSummary;
    ti.exact = false;
    if (kFp8) ti.ks = sc.kt[static_cast<size_t>(h) * ((nkb + 127) / 128) + (t - k - nxt)];
  }
  return ti;
}

// Keys (columns of S, rows of V) the MMAs of a tile cover: exact tiles stop at their valid
// rows rounded up to 16 (the MMA's N step for M = 128), summary tiles cover all 128.
__device__ __forceinline__ int tile_cols(const TileInfo& ti) {
  return ti.exact ? min(128, max(16, (ti.nvalid + 15) & ~15)) : 128;
}

// Reads 64 columns of this thread's S row (TMEM) and turns them into logits: exact tiles give
// raw scores (the scale is applied in the exponent) with columns past the block set to -inf;
// summary tiles give s*sl + offset (offset -inf for selected blocks and padding), sl being the
// logit scale in log2 units (times the FP8 scales).
// Exact tiles: raw scores (the scale is applied in the exponent), columns past the block's
// rows set to -inf.
__device__ __forceinline__ void load_logits_exact(uint32_t taddr, int col0, const TileInfo& ti,
                                                  float (&x)[64]) {
  uint32_t r[64];
  tmem_ld64(taddr, r);
#pragma unroll
  for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(r[j]);
  if (ti.nvalid < col0 + 64) {
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (col0 + j >= ti.nvalid) x[j] = -INFINITY;
  }
}

// Summary tiles: s*sl + offset (offset -inf for selected blocks and padding), sl being the logit
// scale in log2 units (times the FP8 scales).
template <bool kBiasSmem>
__device__ __forceinline__ void load_logits_summary(uint32_t taddr, int col0, const TileInfo& ti,
                                                    float sl, const float* biasrow,
                                                    const float* cb, const uint32_t* selmask,
                                                    int nkb, float (&x)[64]) {
  uint32_t r[64];
  tmem_ld64(taddr, r);
#pragma unroll
  for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(r[j]);
  if (kBiasSmem) {
    const float4* br = reinterpret_cast<const float4*>(biasrow + ti.y + col0);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float4 b = br[j];
      x[4 * j] = fmaf(x[4 * j], sl, b.x);
      x[4 * j + 1] = fmaf(x[4 * j + 1], sl, b.y);
      x[4 * j + 2] = fmaf(x[4 * j + 2], sl, b.z);
      x[4 * j + 3] = fmaf(x[4 * j + 3], sl, b.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const int B = ti.y + col0 + j;
      const int Bc = min(B, nkb - 1);
      const float c = cb[Bc];                         // unconditional: the loads batch up
      const uint32_t bits = selmask[Bc >> 5];
      const bool live = B < nkb && !((bits >> (Bc & 31)) & 1u);
      x[j] = live ? fmaf(x[j], sl, c * kLog2e) : -INFINITY;
    }
  }
}

// Reads 64 columns of this thread's S row (TMEM) and turns them into logits, for a tile of
// either kind (the reference of the first tiles).
template <bool kBiasSmem>
__device__ __forceinline__ void load_logits(uint32_t taddr, int col0, const TileInfo& ti,
                                            float sl, const float* biasrow,
                                            const float* cb, const uint32_t* selmask, int nkb,
                                            float (&x)[64]) {
  if (ti.exact)
    load_logits_exact(taddr, col0, ti, x);
  else
    load_logits_summary<kBiasSmem>(taddr, col0, ti, sl, biasrow, cb, selmask, nkb, x);
}

// The 32 columns col0 .. col0+31 of an exact tile into x[0..31] (columns past the valid rows
// masked to -inf); x[32..63] are left as they are.
__device__ __forceinline__ void load_logits32_exact(uint32_t taddr, int col0, const TileInfo& ti,
                                                    float (&x)[64]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = (col0 + j < ti.nvalid) ? __uint_as_float(r[j]) : -INFINITY;
}

__device__ __forceinline__ float max32(const float (&x)[64]) {
  float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
  for (int j = 4; j < 32; j += 8) {
    mx[0] = fmax3(mx[0], x[j], x[j + 1]);
    mx[1] = fmax3(mx[1], x[j + 2], x[j + 3]);
    mx[2] = fmax3(mx[2], x[j + 4], x[j + 5]);
    mx[3] = fmax3(mx[3], x[j + 6], x[j + 7]);
  }
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
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

// p = 2^(x*c - m) for the 32 columns x[j0 .. j0+31], packed to bf16 pairs; returns their sum.
__device__ __forceinline__ float exp32_at(const float (&x)[64], int j0, float c, float m,
                                          uint32_t (&pk)[16]) {
  const uint64_t c2 = f2_splat(c);
  const uint64_t nm2 = f2_splat(-m);
  uint64_t sum2[2] = {0, 0};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint64_t a2 = f2_fma(f2_pack(x[j0 + 2 * j], x[j0 + 2 * j + 1]), c2, nm2);
    float a0, a1;
    f2_unpack(a2, a0, a1);
    const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
    sum2[j & 1] = f2_add(sum2[j & 1], f2_pack(p0, p1));
    pk[j] = pack_bf16(p0, p1);
  }
  float s0, s1;
  f2_unpack(f2_add(sum2[0], sum2[1]), s0, s1);
  return s0 + s1;
}

}  // namespace

template <int D, bool kBiasSmem, bool kFp8, bool kPersist, bool kRoute, bool kVarTiles>
__global__ void __launch_bounds__(kPersist ? kThreadsFused : kThreads, 1) attend_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kt,
    const __grid_constant__ CUtensorMap map_vt, const __grid_constant__ CUtensorMap map_kc,
    const __grid_constant__ CUtensorMap map_vc, int nc, const float* __restrict__ cbias,
    const int32_t* __restrict__ sel, int kcap, const int32_t* __restrict__ sel_count,
    const int32_t* __restrict__ q_perm,
    const int32_t* __restrict__ q_offsets, int nqb, const int32_t* __restrict__ k_offsets,
    int nkb, int N, void* __restrict__ out, int out_dtype, uint32_t* err, const Fp8Scales sc,
    uint64_t wait_ns, int H, const float* __restrict__ qbar_blocks,
    const float* __restrict__ kbar, int32_t* __restrict__ sel_out) {
  static_assert(!kFp8 || D == 128, "FP8 logits: d = 128 (one 128-byte row per key)");
  static_assert(!kPersist || (kBiasSmem && !kFp8), "persistent CTAs: bf16, bias row in smem");
  static_assert(!kRoute || kPersist, "in-kernel routing runs in persistent CTAs");
  constexpr int QK_BYTES = 128 * D * (kFp8 ? 1 : 2);   // one Q or K tile
  constexpr int V_BYTES = 128 * D * 2;                 // one V tile (bf16)
  constexpr int QK_ATOMS = kFp8 ? 1 : D / 64;          // 128-byte swizzle atoms across a row
  constexpr int V_ATOMS = D / 64;
  constexpr int QK_ATOM_X = kFp8 ? 128 : 64;           // elements per atom row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qst = smem;
  uint8_t* kst = qst + QK_BYTES;
  uint8_t* vst = kst + kKStages * QK_BYTES;
  Barriers* bars = reinterpret_cast<Barriers*>(vst + kVStages * V_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // Per query block: a bit per selected key block and the summary-row offsets in log2 units
  // (-inf for selected blocks and padding; 16-byte aligned: the softmax reads them with float4
  // loads).  With in-kernel routing there are two of each plus the selection itself: the
  // current query block's and the next one's, which the K producer routes meanwhile.
  const int nwords = (nkb + 31) / 32;
  const int nbias = kBiasSmem ? (nkb + 127) / 128 * 128 : 0;
  uint32_t* selmask_b[2];
  float* biasrow_b[2];
  int32_t* sel_s_b[2] = {nullptr, nullptr};
  RouteSmem rsm{nullptr, nullptr, nullptr};
  {
    uint8_t* p = reinterpret_cast<uint8_t*>(tmem_slot + 4);
    auto carve = [&](size_t bytes) {
      p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
      uint8_t* at = p;
      p += bytes;
      return at;
    };
    for (int b = 0; b < (kPersist ? 2 : 1); ++b) {
      selmask_b[b] = reinterpret_cast<uint32_t*>(carve(static_cast<size_t>(nwords) * 4));
      biasrow_b[b] = reinterpret_cast<float*>(carve(static_cast<size_t>(nbias) * 4));
    }
    if (kPersist) {
      for (int b = 0; b < 2; ++b) sel_s_b[b] = reinterpret_cast<int32_t*>(carve(kcap * 4u));
      if (kRoute) {
        rsm.keys = reinterpret_cast<uint32_t*>(carve(static_cast<size_t>(nkb) * 4));
        rsm.hist = reinterpret_cast<uint32_t*>(carve(256 * 4));
        rsm.qn = reinterpret_cast<float*>(carve(D * 4));
      }
    } else {
      selmask_b[1] = selmask_b[0];
      biasrow_b[1] = biasrow_b[0];
    }
  }

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  __shared__ int s_skip, s_rerun;
  // [group][row]: first-tile maxima (the reference), then sums and maxima for the epilogue
  __shared__ float ex_m[2][128], ex_l[2][128], ex_mt[2][128];
  // Query blocks of this CTA: one, (blockIdx.x, blockIdx.y), or with in-kernel routing every
  // gridDim.x-th of the H*nqb (head-major) starting at blockIdx.x.
  const int n_items = kPersist ? H * nqb : 1;
  int item = kPersist ? static_cast<int>(blockIdx.x) : 0;
  if (kPersist && item >= n_items) return;
  const int nxt = (nc + 127) / 128;                 // context tiles

  if (tid == 0) {
    s_skip = launch_timed_out(err) ? 1 : 0;                // an earlier CTA gave up
    s_rerun = 0;
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < kKStages; ++s) mbar_init(&bars->kfull[s], 1);
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bars->sfull[b], 1);
      mbar_init(&bars->pready[b], 4 * 32);
    }
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (s_skip) {                                            // uniform: give back TMEM and leave
    if (warp == 0) tmem_dealloc(*tmem_slot, 512);
    return;
  }
  if (!kPersist && warp < 8) {
    // The selection comes from the routing kernel.  The softmax warps build the mask and the
    // bias row (the only readers) while the producers and the MMA warp already start.
    const int h = blockIdx.y, A = blockIdx.x;
    const int k = sel_count ? max(0, min(sel_count[static_cast<size_t>(h) * nqb + A], kcap)) : kcap;
    const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
    const float* cb = cbias + static_cast<size_t>(h) * nkb;
    for (int i = tid; i < nwords; i += 256) selmask_b[0][i] = 0u;
    if (kBiasSmem)
      for (int i = tid; i < nct * 128; i += 256)
        biasrow_b[0][i] = (i < nkb) ? cb[i] * kLog2e : -INFINITY;
    named_bar_sync(5, 256);
    const int32_t* srow = sel + (static_cast<size_t>(h) * nqb + A) * kcap;
    for (int i = tid; i < k; i += 256) {
      const int B = srow[i];
      if (B >= 0 && B < nkb) {
        atomicOr(&selmask_b[0][B >> 5], 1u << (B & 31));
        if (kBiasSmem) biasrow_b[0][B] = -INFINITY;
      } else {
        flag_error(err, kErrSel);
      }
    }
    named_bar_sync(5, 256);
  }
  // Persistent CTAs: the 12th warp routes this CTA's first query block (selection, mask and
  // bias row) before any tile.
  RouteJob job = route_job_none();
  if (kPersist) {
    if (warp == kWarpRoute) {
      job = route_job(item / nqb, item % nqb, 0);
      while (job.stage != kRjDone)
        route_step<D>(job, rsm, qbar_blocks, kbar, cbias, nqb, nkb, kcap, sel_s_b[0],
                      selmask_b[0], biasrow_b[0], sel_out, lane);
    }
    __syncthreads();
  }
  const uint32_t tbase = *tmem_slot;
  // Barrier phases count over the CTA's whole life: tiles (both passes of every query block),
  // passes (the `done` barrier) and query blocks (the Q tile).
  int tiles_base = 0, passes_base = 0, items_done = 0;
  int issued = 0;                                  // producers: loads issued so far
  for (int cur = 0;; cur ^= 1) {
  const int A = kPersist ? item % nqb : static_cast<int>(blockIdx.x);
  const int h = kPersist ? item / nqb : static_cast<int>(blockIdx.y);
  // selected blocks of this query block: kcap, or its own count (threshold routing) when
  // sel_count is given; rows of sel are kcap apart either way
  const int k = sel_count ? max(0, min(sel_count[static_cast<size_t>(h) * nqb + A], kcap)) : kcap;
  const int nct = (k < nkb) ? (nkb + 127) / 128 : 0;
  const int T = k + nxt + nct;
  const int32_t* sel_row = kPersist ? sel_s_b[cur] : sel + (static_cast<size_t>(h) * nqb + A) * kcap;
  const float* cb = cbias + static_cast<size_t>(h) * nkb;
  const uint32_t* selmask = selmask_b[cur];
  const float* biasrow = biasrow_b[cur];
  const int qlo = q_offsets[A];
  if (kPersist && warp == kWarpRoute) {
    // route the CTA's next query block into the other buffers while this one is attended
    const int nitem = item + static_cast<int>(gridDim.x);
    job = nitem < n_items ? route_job(nitem / nqb, nitem % nqb, cur ^ 1) : route_job_none();
  }

  // Pass 0 exponentiates every tile against a fixed reference per row (the larger of the two
  // groups' first-tile maxima) and records the maximum of every chunk whose sum is out of
  // range.  A CTA with a row whose sum leaves [2^-60, 2^60] runs pass 1 over the same tiles;
  // there the rows out of the window take their recorded maximum as the reference and the
  // others keep pass 0's.  Barrier phases count tiles over both passes.
  float m_true = -INFINITY;                        // softmax threads: row maximum (log2 units)
  float m_ref0 = 0.f;                              //   pass 0's reference of the row
  bool rerun_row = false;                          //   the row left the window in pass 0
  int npasses = 1;
  for (int pass = 0; pass < 2; ++pass) {
    const int tg0 = tiles_base + pass * T;         // tile counter of this pass's first tile
    const uint32_t done_par = static_cast<uint32_t>(passes_base + pass) & 1u;
    if (warp == kWarpK || warp == kWarpV) {
      // ----------------------------------------------------------- TMA producers
      // The whole warp runs the loop (warp-uniform stage indices and coordinates); one elected
      // lane issues the copies.
      constexpr uint32_t kAll = 0xffffffffu;
      const bool is_k = (warp == kWarpK);
      const int stages = is_k ? kKStages : kVStages;
      const int tile_bytes = is_k ? QK_BYTES : V_BYTES;
      const int atoms = is_k ? QK_ATOMS : V_ATOMS;
      const int atom_x = is_k ? QK_ATOM_X : 64;
      uint8_t* ring = is_k ? kst : vst;
      uint64_t* full = is_k ? bars->kfull : bars->vfull;
      // a K stage is free once the S MMA that read it has completed: stage tg % 3 and S
      // buffer tg % 3 belong to the same tile, so sfull also releases the K ring (one
      // commit less per tile for the MMA thread, measured 1.7% faster)
      static_assert(kKStages == 3, "K stages and S buffers must coincide");
      uint64_t* empty = is_k ? bars->sfull : bars->vempty;
      const CUtensorMap* mx = is_k ? &map_k : &map_v;
      const CUtensorMap* mc = is_k ? &map_kc : &map_vc;
      const CUtensorMap* ms = is_k ? &map_kt : &map_vt;
      if (pass == 0) {
        if (elect_one()) {
          tma_prefetch_desc(mx);
          tma_prefetch_desc(ms);
          if (nxt > 0) tma_prefetch_desc(mc);
          if (is_k) {
            tma_prefetch_desc(&map_q);
            mbar_arrive_expect_tx(&bars->qfull, QK_BYTES);
            const int qrow = min(max(qlo, 0), N - 1);   // rows past the block are never stored
            for (int a = 0; a < QK_ATOMS; ++a)
              tma_load_3d(qst + a * 16384, &map_q, &bars->qfull, a * QK_ATOM_X, qrow, h);
          }
        }
        __syncwarp();
      }
      TileInfo next = tile_info<false>(0, k, nxt, nc, sel_row, k_offsets, nkb, N, sc, h);
      for (int t = 0; t < T; ++t) {
        const int tg = tg0 + t;
        const int s = tg % stages;
        const TileInfo ti = next;
        if (tg >= stages &&
            !__all_sync(kAll, mbar_wait(&empty[s], ((tg / stages) - 1) & 1, abort_flag, err,
                                        wait_ns)))
          break;
        if (elect_one()) {
          if (kVarTiles && is_k) bars->kn[s] = static_cast<uint32_t>(tile_cols(ti));   // before the arrive
          mbar_arrive_expect_tx(&full[s], tile_bytes);
          const CUtensorMap* map = ti.src == kSrcVideo ? mx : (ti.src == kSrcContext ? mc : ms);
          for (int a = 0; a < atoms; ++a)
            tma_load_3d(ring + s * tile_bytes + a * 16384, map, &full[s], a * atom_x, ti.y, h);
        }
        __syncwarp();
        issued = tg + 1;
        if (t + 1 < T)
          next = tile_info<false>(t + 1, k, nxt, nc, sel_row, k_offsets, nkb, N, sc, h);
      }
      // every load this pass issued has landed before the pass ends (after an abort some were
      // never consumed; otherwise these phases are complete already and the waits return at once)
      for (int tg = max(tg0, issued - stages); tg < issued; ++tg)
        wait_bounded_ignore_abort(&full[tg % stages], (tg / stages) & 1);
      if (is_k) wait_bounded_ignore_abort(&bars->qfull, items_done & 1);
    } else if (warp == kWarpMma) {
      // ---------------------------------------------------------------- MMA issuer
      // The whole warp runs the issue loop, so stage indices and descriptors are warp-uniform
      // values; one elected lane issues the MMAs and their commits (the same lane each time:
      // the warp is converged at every election, and a commit tracks its own thread's MMAs).
      // the S descriptor without its N field (set per tile)
      constexpr uint32_t idS_base = (kFp8 ? idesc_e4m3(128, 128) : idesc_bf16(128, 128, false, false)) &
                                    ~(0x3Fu << 17);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      constexpr uint32_t kAll = 0xffffffffu;
      // descriptors built once; per MMA only a compile-time offset (16-byte units) changes
      const uint64_t qd = sdesc_sw128(smem_u32(qst), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(kst), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(vst), 16384, 1024);
      bool ok = pass > 0 ||
                __all_sync(kAll, mbar_wait(&bars->qfull, items_done & 1, abort_flag, err, wait_ns));
      // S(t) of this pass into buffer (tg0 + t) % 3
      auto issue_s = [&](int t) -> bool {
        const int tg = tg0 + t;
        const int s = tg % kKStages;
        if (!__all_sync(kAll, mbar_wait(&bars->kfull[s], (tg / kKStages) & 1, abort_flag, err,
                                        wait_ns)))
          return false;
        const uint32_t dcol = tbase + (tg % 3) * 128;
        const uint64_t kd = kdesc0 + static_cast<uint64_t>(s * (QK_BYTES >> 4));
        // variable tiles: S covers the tile's keys only (N = its valid rows rounded up to 16)
        const uint32_t ncols = kVarTiles ? bars->kn[s] : 128u;
        const uint32_t idSn = idS_base | ((ncols >> 3) << 17);
        if (elect_one()) {
          if (kVarTiles) bars->bn[tg % 3] = ncols;
          if constexpr (kFp8) {
            // 32 e4m3 values of d = 32 bytes per MMA, all inside the one 128-byte atom row
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_ss_f8(dcol, qd + kk * 2, kd + kk * 2, idSn, kk > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk / 4) * 16384 + (kk % 4) * 32) / 16;
              mma_ss(dcol, qd + off, kd + off, idSn, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(&bars->sfull[tg % 3]);
        }
        __syncwarp();
        return true;
      };
      for (int t = 0; ok && t < min(T, 3); ++t) ok = issue_s(t);
      for (int t = 0; ok && t < T; ++t) {
        const int tg = tg0 + t;
        if (!__all_sync(kAll, mbar_wait(&bars->pready[tg % 3], (tg / 3) & 1, abort_flag, err,
                                        wait_ns)))
          break;
        tc_fence_after_sync();
        const int s = tg % kVStages;
        if (!__all_sync(kAll, mbar_wait(&bars->vfull[s], (tg / kVStages) & 1, abort_flag, err,
                                        wait_ns)))
          break;
        const uint64_t vd = vdesc0 + static_cast<uint64_t>(s * (V_BYTES >> 4));
        const uint32_t pcol = tbase + (tg % 3) * 128;               // P(t) over S(t)
        if (elect_one()) {
          // the tile's keys only, 16 per MMA (P past them is never read)
          const int nk = kVarTiles ? static_cast<int>(bars->bn[tg % 3] >> 4) : 8;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            if (kk < nk)
              mma_ts(tbase + kColO, pcol + kk * 8, vd + (kk * 2048) / 16, idO,
                     (kk > 0 || t > 0) ? 1u : 0u);
          tc_commit(&bars->vempty[s]);
        }
        __syncwarp();
        // S(t+3) reuses the columns of P(t): issued after PV(t), and MMAs of one thread
        // execute in order
        if (t + 3 < T && !(ok = issue_s(t + 3))) break;
      }
      // every MMA complete: the softmax epilogue reads O, and TMEM is reused or freed after
      if (elect_one()) tc_commit(&bars->done);
      __syncwarp();
      wait_bounded_ignore_abort(&bars->done, done_par);
    } else if (kPersist && warp == kWarpRoute) {
      // ------------------------------------------------------------------ routing warp
      // the next query block's scores and Top-K, while the MMAs and the softmax run this one
      if (pass == 0)
        while (job.stage != kRjDone && !*abort_flag)
          route_step<D>(job, rsm, qbar_blocks, kbar, cbias, nqb, nkb, kcap, sel_s_b[job.buf],
                        selmask_b[job.buf], biasrow_b[job.buf], sel_out, lane);
    } else if (warp < 8) {
      // ---------------------------------------------------------------- softmax rows
      const int q4 = warp & 3, grp = warp >> 2;          // row quarter, tile group
      const int row = q4 * 32 + lane;                    // 0..127 == TMEM lane
      const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
      // logit scale in log2 units; FP8 queries carry their block's scale
      const float scale_log2 = kLog2e * rsqrtf(static_cast<float>(D)) *
                               (kFp8 ? sc.q[static_cast<size_t>(h) * nqb + A] : 1.f);
      float l_run = 0.f;
      bool ok = true;
      float x[64];
      float m_ref;
      if (pass == 0) {
        // reference: the row maximum of the first tile of each group, shared by both
        float mt = -INFINITY;
        if (grp < T) {
          const int tg = tg0 + grp;
          const TileInfo ti = tile_info<kFp8>(grp, k, nxt, nc, sel_row, k_offsets, nkb, N, sc, h);
          const float tsl = scale_log2 * ti.ks;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars->sfull[tg % 3], (tg / 3) & 1, abort_flag, err, wait_ns));
          if (ok) {
            tc_fence_after_sync();
            const uint32_t sbuf = tbase + lane_off + (tg % 3) * 128;
            load_logits<kBiasSmem>(sbuf, 0, ti, tsl, biasrow, cb, selmask, nkb, x);
            mt = max64(x);
            load_logits<kBiasSmem>(sbuf + 64, 64, ti, tsl, biasrow, cb, selmask, nkb, x);
            mt = fmaxf(mt, max64(x));
            if (ti.exact) mt *= tsl;
          }
        }
        ex_m[grp][row] = mt;
        named_bar_sync(1 + q4, 64);                      // the two groups of this quarter
        m_ref = fmaxf(ex_m[0][row], ex_m[1][row]);
      } else {
        // rows that left the window take the recorded maximum (both groups' maxima, merged in
        // the epilogue); the others keep the reference that served them
        m_ref = rerun_row ? m_true : m_ref0;
      }
      if (!(m_ref > -INFINITY)) m_ref = 0.f;
      if (pass == 0) m_ref0 = m_ref;
      TileInfo next = tile_info<kFp8>(grp, k, nxt, nc, sel_row, k_offsets, nkb, N, sc, h);
      // One tile of this group; the exact tiles (selected blocks, then context rows) come
      // before the summary tiles, so each kind runs in a loop of its own that carries only its
      // own logit path.
      // kind: 1 exact, 2 summary, 0 either (decided per tile)
      auto tile = [&](int t, auto kind) -> bool {
        constexpr int kKind = decltype(kind)::value;
        const TileInfo ti = next;
        const int tg = tg0 + t;
        const int b = tg % 3;
        if (pass > 0 || t >= 2) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait(&bars->sfull[b], (tg / 3) & 1, abort_flag, err, wait_ns)))
            return false;
          tc_fence_after_sync();
        }
        if (t + 2 < T)
          next = tile_info<kFp8>(t + 2, k, nxt, nc, sel_row, k_offsets, nkb, N, sc, h);
        const uint32_t sbuf = tbase + lane_off + b * 128;
        const float tsl = scale_log2 * ti.ks;
        const bool exact = kKind == 1 || (kKind == 0 && ti.exact);
        const float c = exact ? tsl : 1.f;
        // The row maximum is only needed for a repeat, and only to within a few units: a
        // chunk whose sum stays in [2^-40, 2^40] has its maximum within 40 of the reference
        // and cannot drive the row sum out of [2^-60, 2^60] (fewer than 2^16 chunks per row),
        // so only chunks outside that range (rare) take their maximum.
        // only the columns the MMAs covered (exact tiles: the valid rows rounded up to 16)
        const int ncols = (kVarTiles && kKind != 2) ? tile_cols(ti) : 128;
        float rowsum = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half == 1 && ncols <= 64) break;
          uint32_t p16[16];
          float cs;
          if (half == 1 && ncols <= 96) {
            load_logits32_exact(sbuf + 64, 64, ti, x);      // exact tiles only (summary: 128)
            cs = exp32_at(x, 0, c, m_ref, p16);
            tmem_st16_issue(sbuf + 32, p16);
            if (!(cs >= 0x1p-40f && cs <= 0x1p40f)) m_true = fmaxf(m_true, max32(x) * tsl);
          } else {
            if constexpr (kKind == 1)
              load_logits_exact(sbuf + half * 64, half * 64, ti, x);
            else if constexpr (kKind == 2)
              load_logits_summary<kBiasSmem>(sbuf + half * 64, half * 64, ti, tsl, biasrow, cb,
                                             selmask, nkb, x);
            else
              load_logits<kBiasSmem>(sbuf + half * 64, half * 64, ti, tsl, biasrow, cb, selmask,
                                     nkb, x);
            cs = exp32_at(x, 0, c, m_ref, p16);
            tmem_st16_issue(sbuf + half * 32, p16);
            cs += exp32_at(x, 32, c, m_ref, p16);
            tmem_st16_issue(sbuf + half * 32 + 16, p16);
            if (!(cs >= 0x1p-40f && cs <= 0x1p40f)) {
              const float mt = max64(x);
              m_true = fmaxf(m_true, exact ? mt * tsl : mt);
            }
          }
          rowsum += cs;
        }
        l_run += rowsum;
        tmem_wait_st();                                 // P complete before it is signalled
        tc_fence_before_sync();
        mbar_arrive(&bars->pready[b]);
        return true;
      };
      int t = grp;
      if constexpr (kFp8 || kPersist) {
        // one loop (split, these instantiations spill more registers)
        for (; ok && t < T; t += 2) ok = tile(t, std::integral_constant<int, 0>{});
      } else {
        const int t_exact = k + nxt;                     // tiles before the summary tiles
        for (; ok && t < T && t < t_exact; t += 2) ok = tile(t, std::integral_constant<int, 1>{});
        for (; ok && t < T; t += 2) ok = tile(t, std::integral_constant<int, 2>{});
      }
      // ---- epilogue: O / (l_0 + l_1), scattered to the original token order
      bool fine = ok && T > 0;
      if (fine) fine = __all_sync(0xffffffffu, mbar_wait(&bars->done, done_par, abort_flag, err, wait_ns));
      ex_l[grp][row] = l_run;
      ex_mt[grp][row] = m_true;
      named_bar_sync(1 + q4, 64);
      const float l_tot = ex_l[0][row] + ex_l[1][row];
      m_true = fmaxf(ex_mt[0][row], ex_mt[1][row]);
      if (fine) {
        tc_fence_after_sync();
        const int qsize = max(0, min(q_offsets[A + 1] - qlo, kMaxBlock));
        // a sum outside the window means the reference was far from the row maximum
        if (pass == 0 && row < qsize && !(l_tot >= 0x1p-60f && l_tot <= 0x1p60f)) {
          s_rerun = 1;
          rerun_row = true;
        }
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        int tok = -1;
        if (row < qsize) {
          tok = q_perm[static_cast<size_t>(h) * N + qlo + row];
          if (tok < 0 || tok >= N) {
            if (grp == 0) flag_error(err, kErrPerm);
            tok = -1;
          }
        }
        // each group's warp writes half of the d output columns
        constexpr int HALF = D / 2;
#pragma unroll
        for (int cc = 0; cc < HALF / 32; ++cc) {
          const int col = grp * HALF + cc * 32;
          uint32_t a[32];
          tmem_ld32(tbase + lane_off + kColO + col, a);
          float o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(a[j]) * inv;
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
    // every role is done with this pass (TMEM reads included) before the next one starts
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (pass == 1 || !s_rerun || *abort_flag) break;   // uniform: written before the barrier
    npasses = 2;
  }
  tiles_base += npasses * T;
  passes_base += npasses;
  ++items_done;
  if (!kPersist) break;
  // the next query block's routing completes before it starts
  if (kPersist && warp == kWarpRoute)
    while (job.stage != kRjDone && !*abort_flag)
      route_step<D>(job, rsm, qbar_blocks, kbar, cbias, nqb, nkb, kcap, sel_s_b[job.buf],
                    selmask_b[job.buf], biasrow_b[job.buf], sel_out, lane);
  if (tid == 0) {
    s_rerun = 0;
    s_skip = launch_timed_out(err) ? 1 : 0;
  }
  __syncthreads();
  item += static_cast<int>(gridDim.x);
  if (*abort_flag || s_skip || item >= n_items) break;   // uniform: written before the barrier
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

static size_t align16(size_t b) { return (b + 15) & ~static_cast<size_t>(15); }

// Dynamic shared memory of a launch: 1 KB of alignment slack, the Q tile, the K and V rings,
// the barriers, then (16-byte aligned each) the selection mask and bias row of one query block,
// or with in-kernel routing two of each plus two selections, the routing keys, a histogram and
// the query-block mean.
static size_t attend_smem_bytes(int d, int nkb, int k, bool fp8, bool persist = false,
                                bool route = false) {
  const size_t qk = static_cast<size_t>(128) * d * (fp8 ? 1 : 2);
  const size_t v = static_cast<size_t>(128) * d * 2;
  const size_t words = static_cast<size_t>((nkb + 31) / 32) * 4;
  const size_t bias = bias_in_smem(nkb, k) || persist
                          ? static_cast<size_t>((nkb + 127) / 128) * 128 * 4 : 0;
  size_t b = 1024 + (1 + kKStages) * qk + kVStages * v + sizeof(Barriers) + 16;
  const int nbuf = persist ? 2 : 1;
  b += nbuf * (align16(words) + 16 + align16(bias) + 16);
  if (persist) b += 2 * (align16(static_cast<size_t>(k) * 4) + 16);
  if (route) b += align16(static_cast<size_t>(nkb) * 4) + 16 + 256 * 4 + 16 + d * 4 + 16;
  return b;
}

constexpr size_t kSmemLimit = 232448;   // 227 KB of opt-in shared memory per CTA

// All key blocks hold exactly 128 tokens (sizes are 1..128 and sum to N) - then every exact
// tile is a full MMA tile and the kernel without per-tile widths runs.
static bool all_blocks_full(int N, int nkb) { return static_cast<long long>(nkb) * 128 == N; }

static cudaError_t persistent_grid(long long items, int* grid) {
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  *grid = static_cast<int>(items < nsm ? items : nsm);   // one persistent CTA per SM
  return e;
}

template <int D, bool kBiasSmem, bool kFp8, bool kVar>
static cudaError_t launch_attend_t(const AttendMaps& m, int nc, const float* cbias,
                                   const int32_t* sel, int k, const int32_t* sel_count,
                                   const int32_t* q_perm, const int32_t* q_offsets,
                                   int nqb, const int32_t* k_offsets, int nkb, int H, int N,
                                   void* out, int out_dtype, uint32_t* err, const Fp8Scales& sc,
                                   cudaStream_t s) {
  // with per-row counts any row may have summary tiles: size for k < nkb
  const size_t smem = attend_smem_bytes(D, nkb, sel_count ? 0 : k, kFp8);
  auto kern = attend_kernel<D, kBiasSmem, kFp8, false, false, kVar>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(nqb, H);
  kern<<<grid, kThreads, smem, s>>>(m.q, m.k, m.v, m.kt, m.vt, m.kc, m.vc, nc, cbias, sel, k,
                                    sel_count, q_perm, q_offsets, nqb, k_offsets, nkb, N, out,
                                    out_dtype, err, sc, wait_limit_ns(), H, nullptr, nullptr,
                                    nullptr);
  return cudaGetLastError();
}

template <int D, bool kBiasSmem, bool kFp8>
static cudaError_t launch_attend_v(const AttendMaps& m, int nc, const float* cbias,
                                   const int32_t* sel, int k, const int32_t* sel_count,
                                   const int32_t* q_perm, const int32_t* q_offsets,
                                   int nqb, const int32_t* k_offsets, int nkb, int H, int N,
                                   void* out, int out_dtype, uint32_t* err, const Fp8Scales& sc,
                                   cudaStream_t s) {
  return all_blocks_full(N, nkb)
             ? launch_attend_t<D, kBiasSmem, kFp8, false>(m, nc, cbias, sel, k, sel_count, q_perm,
                                                          q_offsets, nqb, k_offsets, nkb, H, N,
                                                          out, out_dtype, err, sc, s)
             : launch_attend_t<D, kBiasSmem, kFp8, true>(m, nc, cbias, sel, k, sel_count, q_perm,
                                                         q_offsets, nqb, k_offsets, nkb, H, N,
                                                         out, out_dtype, err, sc, s);
}

cudaError_t launch_attend(const AttendMaps& maps, int nc, const float* cbias,
                          const int32_t* sel, int k, const int32_t* q_perm,
                          const int32_t* q_offsets, int nqb, const int32_t* k_offsets, int nkb,
                          int H, int N, int d, void* out, int out_dtype, uint32_t* err,
                          cudaStream_t s, const int32_t* sel_count) {
  const bool bs = bias_in_smem(nkb, sel_count ? 0 : k);
  const Fp8Scales none{nullptr, nullptr, nullptr, nullptr};
  if (d == 128)
    return bs ? launch_attend_v<128, true, false>(maps, nc, cbias, sel, k, sel_count, q_perm,
                                                  q_offsets, nqb, k_offsets, nkb, H, N, out,
                                                  out_dtype, err, none, s)
              : launch_attend_v<128, false, false>(maps, nc, cbias, sel, k, sel_count, q_perm,
                                                   q_offsets, nqb, k_offsets, nkb, H, N, out,
                                                   out_dtype, err, none, s);
  return bs ? launch_attend_v<64, true, false>(maps, nc, cbias, sel, k, sel_count, q_perm,
                                               q_offsets, nqb, k_offsets, nkb, H, N, out,
                                               out_dtype, err, none, s)
            : launch_attend_v<64, false, false>(maps, nc, cbias, sel, k, sel_count, q_perm,
                                                q_offsets, nqb, k_offsets, nkb, H, N, out,
                                                out_dtype, err, none, s);
}

cudaError_t launch_attend_fp8(const AttendMaps& maps, const float* q_scale,
                              const float* k_scale, const float* kt_scale,
                              const float* kc_scale, int nc, const float* cbias,
                              const int32_t* sel, int k, const int32_t* q_perm,
                              const int32_t* q_offsets, int nqb, const int32_t* k_offsets,
                              int nkb, int H, int N, void* out, int out_dtype, uint32_t* err,
                              cudaStream_t s) {
  const Fp8Scales sc{q_scale, k_scale, kt_scale, kc_scale};
  return bias_in_smem(nkb, k)
             ? launch_attend_v<128, true, true>(maps, nc, cbias, sel, k, nullptr, q_perm,
                                                q_offsets, nqb, k_offsets, nkb, H, N, out,
                                                out_dtype, err, sc, s)
             : launch_attend_v<128, false, true>(maps, nc, cbias, sel, k, nullptr, q_perm,
                                                 q_offsets, nqb, k_offsets, nkb, H, N, out,
                                                 out_dtype, err, sc, s);
}

bool attend_fused_supported(int d, int nkb, int k) {
  return d == 128 && k < nkb && bias_in_smem(nkb, k) &&
         attend_smem_bytes(d, nkb, k, false, true, true) <= kSmemLimit;
}

template <bool kVar>
static cudaError_t launch_fused_t(const AttendMaps& m, int nc, const float* cbias,
                                  const float* qbar_blocks, const float* kbar, int k,
                                  const int32_t* q_perm, const int32_t* q_offsets, int nqb,
                                  const int32_t* k_offsets, int nkb, int H, int N, void* out,
                                  int out_dtype, uint32_t* err, int32_t* sel_out,
                                  cudaStream_t s) {
  const size_t smem = attend_smem_bytes(128, nkb, k, false, true, true);
  auto kern = attend_kernel<128, true, false, true, true, kVar>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = 0;
  if ((e = persistent_grid(static_cast<long long>(H) * nqb, &grid)) != cudaSuccess) return e;
  const Fp8Scales none{nullptr, nullptr, nullptr, nullptr};
  kern<<<grid, kThreadsFused, smem, s>>>(m.q, m.k, m.v, m.kt, m.vt, m.kc, m.vc, nc, cbias, nullptr, k,
                                    nullptr, q_perm, q_offsets, nqb, k_offsets, nkb, N, out,
                                    out_dtype, err, none, wait_limit_ns(), H, qbar_blocks, kbar,
                                    sel_out);
  return cudaGetLastError();
}

cudaError_t launch_attend_fused(const AttendMaps& maps, int nc, const float* cbias,
                                const float* qbar_blocks, const float* kbar, int k,
                                const int32_t* q_perm, const int32_t* q_offsets, int nqb,
                                const int32_t* k_offsets, int nkb, int H, int N, int d, void* out,
                                int out_dtype, uint32_t* err, int32_t* sel_out, cudaStream_t s) {
  if (!attend_fused_supported(d, nkb, k)) return cudaErrorInvalidValue;
  return all_blocks_full(N, nkb)
             ? launch_fused_t<false>(maps, nc, cbias, qbar_blocks, kbar, k, q_perm, q_offsets,
                                     nqb, k_offsets, nkb, H, N, out, out_dtype, err, sel_out, s)
             : launch_fused_t<true>(maps, nc, cbias, qbar_blocks, kbar, k, q_perm, q_offsets,
                                    nqb, k_offsets, nkb, H, N, out, out_dtype, err, sel_out, s);
}

}  // namespace spark
