// Block scoring + Top-K of ONE query block by one warp, in short bounded steps: the attention
// kernel's routing warp runs them for the next query block while the current one is attended,
// and the selection never leaves shared memory (Spark-H3 blog, "Discussion": blocks scored from
// block-level means; "Spark-Reblock": a fixed Top-K budget).
//
// The arithmetic is that of route_kernel (route.cu): each score is a sequential fp32 FMA over
// d of the query-block mean and the key-block mean, starting from 0, the positive factor
// 1/sqrt(d) left out; scores are ordered as order-preserving uint32 keys; the k largest are
// selected by an exact radix select (8-bit digits, most significant first), ties to the
// smaller block index, stored ascending.  The selection is therefore the routing kernel's, bit
// for bit.
#pragma once

#include "spark_kernels.cuh"

namespace spark {

// Stages of the job, in order.  Every call does one short step of the current stage.
enum RouteStage : int {
  kRjLoad = 0,    // query-block mean into shared memory, selection mask cleared
  kRjScore,       // 32 key blocks scored per step
  kRjHist,        // histogram of one radix digit, 256 keys per step
  kRjScan,        // the digit of the k-th largest key; next digit or done
  kRjWrite,       // the selection, 256 keys per step, ascending
  kRjBias,        // the bias row of the summary tiles, 512 columns per step
  kRjDone
};

struct RouteJob {
  int stage;
  int pos;            // next key block (or column) of the current stage
  int shift;          // digit being resolved
  uint32_t prefix, pmask;
  int need;           // keys still to take among those matching prefix
  int taken, eq_seen; // selection written so far / keys equal to the threshold seen so far
  int h, A;           // the query block being routed
  int buf;            // destination buffer index
};

__device__ __forceinline__ RouteJob route_job(int h, int A, int buf) {
  return RouteJob{kRjLoad, 0, 24, 0u, 0u, 0, 0, 0, h, A, buf};
}

__device__ __forceinline__ RouteJob route_job_none() {
  return RouteJob{kRjDone, 0, 0, 0u, 0u, 0, 0, 0, 0, 0, 0};
}

__device__ __forceinline__ uint32_t rj_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Shared-memory state of the job: the query-block mean, the row's keys, a 256-bin histogram.
struct RouteSmem {
  float* qn;          // [D]
  uint32_t* keys;     // [nkb]
  uint32_t* hist;     // [256]
};

// One step of the job (all 32 lanes of the calling warp, converged).  When the job completes:
// sel_s holds the k selected ids ascending, selmask a bit per selected block, biasrow the
// nct*128 summary offsets in log2 units (-inf for selected blocks and padding), and sel_out
// (optional) a global copy of the selection.
template <int D>
__device__ __forceinline__ void route_step(RouteJob& j, const RouteSmem& rs,
                                           const float* __restrict__ qbar_blocks,
                                           const float* __restrict__ kbar,
                                           const float* __restrict__ cbias, int nqb, int nkb,
                                           int k, int32_t* sel_s, uint32_t* selmask,
                                           float* biasrow, int32_t* sel_out, int lane) {
  constexpr uint32_t kAll = 0xffffffffu;
  constexpr float kLog2eRj = 1.4426950408889634f;
  switch (j.stage) {
    case kRjLoad: {
      const float* q = qbar_blocks + (static_cast<size_t>(j.h) * nqb + j.A) * D;
      for (int e = lane; e < D; e += 32) rs.qn[e] = q[e];
      for (int i = lane; i < (nkb + 31) / 32; i += 32) selmask[i] = 0u;
      __syncwarp();
      j.stage = kRjScore;
      j.pos = 0;
      return;
    }
    case kRjScore: {
      // 32 key blocks, one per lane; kbar is d-major, so each load is one coalesced row
      const int B = j.pos + lane;
      const float* kb = kbar + static_cast<size_t>(j.h) * D * nkb + min(B, nkb - 1);
      float acc = 0.f;
      constexpr int kE = D;                      // loads in flight per lane (one round trip)
#pragma unroll 1
      for (int e0 = 0; e0 < D; e0 += kE) {
        float v[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) v[e] = __ldg(kb + static_cast<size_t>(e0 + e) * nkb);
#pragma unroll
        for (int e = 0; e < kE; ++e) acc = fmaf(rs.qn[e0 + e], v[e], acc);
      }
      if (B < nkb) rs.keys[B] = rj_order_key(acc);
      __syncwarp();
      j.pos += 32;
      if (j.pos >= nkb) {
        j.pos = 0;
        j.need = k;
        j.stage = k >= nkb ? kRjWrite : kRjHist;   // k >= nkb: every block is taken
      }
      return;
    }
    case kRjHist: {
      if (j.pos == 0) {
        for (int i = lane; i < 256; i += 32) rs.hist[i] = 0u;
        __syncwarp();
      }
      const int end = min(nkb, j.pos + 256);
      for (int B = j.pos + lane; B < end; B += 32) {
        const uint32_t u = rs.keys[B];
        if ((u & j.pmask) == j.prefix) atomicAdd(&rs.hist[(u >> j.shift) & 255u], 1u);
      }
      __syncwarp();
      j.pos = end;
      if (j.pos >= nkb) j.stage = kRjScan;
      return;
    }
    case kRjScan: {
      // lane l owns digits [8l, 8l+8); suffix sums give count(digit >= x)
      uint32_t c[8], local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = rs.hist[lane * 8 + q];
        local += c[q];
      }
      uint32_t suf = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(kAll, suf, off);
        if (lane + off < 32) suf += v;
      }
      uint32_t above = suf - local;
      int best = -1;
      uint32_t best_gt = 0;
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        const uint32_t ge = above + c[q];
        if (best < 0 && ge >= static_cast<uint32_t>(j.need)) {
          best = lane * 8 + q;
          best_gt = above;
        }
        above = ge;
      }
      // the digit of the k-th largest key: the largest x with count(>= x) >= need
      const int dd = __reduce_max_sync(kAll, best);
      const uint32_t gt = __shfl_sync(kAll, best_gt, dd / 8);
      j.need -= static_cast<int>(gt);
      j.prefix |= static_cast<uint32_t>(dd) << j.shift;
      j.pmask |= 255u << j.shift;
      // every key left under the prefix is needed: the remaining digits cannot change the set
      const bool all_taken = static_cast<uint32_t>(j.need) == rs.hist[dd];
      __syncwarp();
      j.pos = 0;
      if (all_taken || j.shift == 0) {
        j.stage = kRjWrite;
        j.taken = 0;
        j.eq_seen = 0;
      } else {
        j.shift -= 8;
        j.stage = kRjHist;
      }
      return;
    }
    case kRjWrite: {
      // keys compared on the resolved digits: above the prefix taken, equal to it taken in
      // ascending block order until `need`, below it left
      const uint32_t lt = (1u << lane) - 1u;
      const int end = min(nkb, j.pos + 256);
      for (int B0 = j.pos; B0 < end; B0 += 32) {
        const int B = B0 + lane;
        const bool valid = B < end;
        const uint32_t u = (valid ? rs.keys[B] : 0u) & j.pmask;
        const bool gt = valid && (k >= nkb || u > j.prefix);
        const bool eq = valid && k < nkb && u == j.prefix;
        const uint32_t eqb = __ballot_sync(kAll, eq);
        const bool take = gt || (eq && j.eq_seen + __popc(eqb & lt) < j.need);
        const uint32_t tb = __ballot_sync(kAll, take);
        if (take) {
          const int at = j.taken + __popc(tb & lt);
          sel_s[at] = B;
          if (sel_out != nullptr) sel_out[(static_cast<size_t>(j.h) * nqb + j.A) * k + at] = B;
        }
        if (lane == 0) selmask[B0 >> 5] = tb;     // B0 is a multiple of 32
        j.taken += __popc(tb);
        j.eq_seen += __popc(eqb);
      }
      __syncwarp();
      j.pos = end;
      if (j.pos >= nkb) {
        j.pos = 0;
        j.stage = (biasrow != nullptr && k < nkb) ? kRjBias : kRjDone;
      }
      return;
    }
    case kRjBias: {
      const float* cb = cbias + static_cast<size_t>(j.h) * nkb;
      const int ncols = (nkb + 127) / 128 * 128;
      const int end = min(ncols, j.pos + 512);
      for (int i = j.pos + lane; i < end; i += 32) {
        const bool live = i < nkb && !((selmask[i >> 5] >> (i & 31)) & 1u);
        biasrow[i] = live ? cb[i] * kLog2eRj : -INFINITY;
      }
      __syncwarp();
      j.pos = end;
      if (j.pos >= ncols) j.stage = kRjDone;
      return;
    }
    default:
      return;
  }
}

}  // namespace spark
