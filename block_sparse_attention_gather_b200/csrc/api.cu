// C ABI of the library (include/spark_bsa.h): argument checks, workspace layout, TMA
// descriptor encoding and the launch sequence of the forward pass.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>

#include "../../include/spark_bsa.h"
#include "spark_kernels.cuh"

using namespace spark;

namespace spark {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 3-D bf16 tensor [H][rows][d] with a 128-row x 64-column box and 128-byte swizzle.
bool encode_rows_map(CUtensorMap* m, const void* base, int H, int rows, int d) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(H)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D e4m3 (byte) tensor [H][rows][d] with a 128-row x 128-byte box and 128-byte swizzle.
bool encode_rows_map_u8(CUtensorMap* m, const void* base, int H, int rows, int d) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(H)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Process-wide limit of the kernels' bounded waits (nanoseconds), read at each launch.
static std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace spark

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int topk_count(int nkb, double ratio) {
  if (nkb < 1 || !(ratio > 0.0) || !(ratio <= 1.0)) return -1;
  double kk = std::ceil(ratio * static_cast<double>(nkb) - 1e-9);
  int k = static_cast<int>(kk);
  if (k < 1) k = 1;
  if (k > nkb) k = nkb;
  return k;
}

spark_status check_sizes(int H, int N, int d, int nqb, int nkb) {
  if (H < 1 || N < 1 || nqb < 1 || nkb < 1 || nqb > N || nkb > N) return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (H > 65535 || nkb > kMaxNkb) return SPARK_ERR_UNSUPPORTED;
  return SPARK_OK;
}

spark_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA; }

spark_status layout_of(int H, int N, int d, int nqb, int nkb, double ratio,
                       spark_bsa_layout* L) {
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  const int k = topk_count(nkb, ratio);
  if (k < 0) return SPARK_ERR_INVALID_ARG;
  const size_t hnd = static_cast<size_t>(H) * N * d;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  L->Qp = take(hnd * 2);
  L->Kp = take(hnd * 2);
  L->Vp = take(hnd * 2);
  L->qbar_blocks = take(static_cast<size_t>(H) * nqb * d * 4);
  L->qbar = take(static_cast<size_t>(H) * d * 4);
  L->kbar = take(static_cast<size_t>(H) * nkb * d * 4);
  L->k_tilde = take(static_cast<size_t>(H) * nkb * d * 2);
  L->v_tilde = take(static_cast<size_t>(H) * nkb * d * 2);
  L->cbias = take(static_cast<size_t>(H) * nkb * 4);
  L->sel = take(static_cast<size_t>(H) * nqb * k * 4);
  L->err = take(4);
  L->total = off;
  L->k = k;
  return SPARK_OK;
}

// Bytes of one bf16 context tensor [H,nc,d] inside a workspace (256-byte aligned).
size_t context_bytes(int H, int nc, int d) {
  return align_up(static_cast<size_t>(H) * static_cast<size_t>(nc) * d * 2);
}

spark_status attend_impl(const void* Qp, const void* Kp, const void* Vp, const void* k_tilde,
                         const void* v_tilde, const float* cbias, const int32_t* sel, int k,
                         const void* Kc, const void* Vc, int nc, const int32_t* q_perm,
                         const int32_t* q_offsets, int nqb, const int32_t* k_offsets, int nkb,
                         int H, int N, int d, void* out, int out_dtype, uint32_t* err,
                         cudaStream_t s, const int32_t* sel_count = nullptr) {
  AttendMaps maps;
  if (!encode_rows_map(&maps.q, Qp, H, N, d) || !encode_rows_map(&maps.k, Kp, H, N, d) ||
      !encode_rows_map(&maps.v, Vp, H, N, d) || !encode_rows_map(&maps.kt, k_tilde, H, nkb, d) ||
      !encode_rows_map(&maps.vt, v_tilde, H, nkb, d))
    return SPARK_ERR_CUDA;
  if (nc > 0) {
    if (!encode_rows_map(&maps.kc, Kc, H, nc, d) || !encode_rows_map(&maps.vc, Vc, H, nc, d))
      return SPARK_ERR_CUDA;
  } else {
    maps.kc = maps.k;                            // never loaded: the kernel has no context tile
    maps.vc = maps.v;
  }
  return from_cuda(launch_attend(maps, nc, cbias, sel, k, q_perm, q_offsets, nqb, k_offsets, nkb,
                                 H, N, d, out, out_dtype, err, s, sel_count));
}

// The attention with the routing inside: the selection of every query block is computed by the
// kernel from the block means (sel_out receives a copy when not null).
spark_status attend_fused_impl(const void* Qp, const void* Kp, const void* Vp,
                               const void* k_tilde, const void* v_tilde, const float* cbias,
                               const float* qbar_blocks, const float* kbar, int k,
                               const void* Kc, const void* Vc, int nc, const int32_t* q_perm,
                               const int32_t* q_offsets, int nqb, const int32_t* k_offsets,
                               int nkb, int H, int N, int d, void* out, int out_dtype,
                               uint32_t* err, int32_t* sel_out, cudaStream_t s) {
  if (!attend_fused_supported(d, nkb, k)) return SPARK_ERR_UNSUPPORTED;
  AttendMaps maps;
  if (!encode_rows_map(&maps.q, Qp, H, N, d) || !encode_rows_map(&maps.k, Kp, H, N, d) ||
      !encode_rows_map(&maps.v, Vp, H, N, d) || !encode_rows_map(&maps.kt, k_tilde, H, nkb, d) ||
      !encode_rows_map(&maps.vt, v_tilde, H, nkb, d))
    return SPARK_ERR_CUDA;
  if (nc > 0) {
    if (!encode_rows_map(&maps.kc, Kc, H, nc, d) || !encode_rows_map(&maps.vc, Vc, H, nc, d))
      return SPARK_ERR_CUDA;
  } else {
    maps.kc = maps.k;                            // never loaded: the kernel has no context tile
    maps.vc = maps.v;
  }
  return from_cuda(launch_attend_fused(maps, nc, cbias, qbar_blocks, kbar, k, q_perm, q_offsets,
                                       nqb, k_offsets, nkb, H, N, d, out, out_dtype, err, sel_out,
                                       s));
}

// FP8 logits: e4m3 Qp8/Kp8/kt8/Kc8 with their group scales, bf16 values.
spark_status attend_fp8_impl(const void* Qp8, const float* q_scale, const void* Kp8,
                             const float* k_scale, const void* Vp, const void* kt8,
                             const float* kt_scale, const void* v_tilde, const float* cbias,
                             const int32_t* sel, int k, const void* Kc8, const float* kc_scale,
                             const void* Vc, int nc, const int32_t* q_perm,
                             const int32_t* q_offsets, int nqb, const int32_t* k_offsets,
                             int nkb, int H, int N, int d, void* out, int out_dtype,
                             uint32_t* err, cudaStream_t s) {
  AttendMaps maps;
  if (!encode_rows_map_u8(&maps.q, Qp8, H, N, d) || !encode_rows_map_u8(&maps.k, Kp8, H, N, d) ||
      !encode_rows_map(&maps.v, Vp, H, N, d) || !encode_rows_map_u8(&maps.kt, kt8, H, nkb, d) ||
      !encode_rows_map(&maps.vt, v_tilde, H, nkb, d))
    return SPARK_ERR_CUDA;
  if (nc > 0) {
    if (!encode_rows_map_u8(&maps.kc, Kc8, H, nc, d) || !encode_rows_map(&maps.vc, Vc, H, nc, d))
      return SPARK_ERR_CUDA;
  } else {
    maps.kc = maps.k;                            // never loaded: the kernel has no context tile
    maps.vc = maps.v;
  }
  return from_cuda(launch_attend_fp8(maps, q_scale, k_scale, kt_scale, kc_scale, nc, cbias, sel,
                                     k, q_perm, q_offsets, nqb, k_offsets, nkb, H, N, out,
                                     out_dtype, err, s));
}

// Byte offsets of the FP8 operands and scales of spark_bsa_forward_fp8 (from the start of
// their region, 256-byte aligned).
struct Fp8Layout {
  size_t Qp8, Kp8, kt8, Kc8, q_scale, k_scale, kt_scale, kc_scale, total;
};

Fp8Layout fp8_layout(int H, int N, int d, int nqb, int nkb, int nc) {
  Fp8Layout F;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t h = static_cast<size_t>(H);
  F.Qp8 = take(h * N * d);
  F.Kp8 = take(h * N * d);
  F.kt8 = take(h * nkb * d);
  F.Kc8 = take(h * nc * d);
  F.q_scale = take(h * nqb * 4);
  F.k_scale = take(h * nkb * 4);
  F.kt_scale = take(h * ((nkb + 127) / 128) * 4);
  F.kc_scale = take(h * ((nc + 127) / 128) * 4);
  F.total = off;
  return F;
}

spark_status check_context(const void* Kc, const void* Vc, int nc) {
  if (nc < 0 || nc > SPARK_MAX_NC) return SPARK_ERR_INVALID_ARG;
  if (nc > 0 && (!Kc || !Vc || !aligned(Kc, 16) || !aligned(Vc, 16)))
    return SPARK_ERR_INVALID_ARG;
  return SPARK_OK;
}

// The whole forward pass; nc == 0 runs without context rows.
spark_status forward_impl(const void* Q, const void* K, const void* V, const void* Kc,
                          const void* Vc, int nc, int dtype, int H, int N, int d,
                          const int32_t* q_perm, const int32_t* k_perm,
                          const int32_t* q_block_offsets, int nqb,
                          const int32_t* k_block_offsets, int nkb, double topk_ratio, void* out,
                          void* workspace, size_t workspace_bytes, cudaStream_t s,
                          bool fp8 = false, bool fused = false) {
  if (!Q || !K || !V || !q_perm || !k_perm || !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_bsa_layout L;
  spark_status st = layout_of(H, N, d, nqb, nkb, topk_ratio, &L);
  if (st != SPARK_OK) return st;
  st = check_context(Kc, Vc, nc);
  if (st != SPARK_OK) return st;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  if (fp8 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (fused && (fp8 || !attend_fused_supported(d, nkb, L.k))) return SPARK_ERR_UNSUPPORTED;
  const size_t cbytes = nc > 0 ? context_bytes(H, nc, d) : 0;
  const size_t fp8_bytes = fp8 ? fp8_layout(H, N, d, nqb, nkb, nc).total : 0;
  if (workspace == nullptr || workspace_bytes < L.total + 2 * cbytes + fp8_bytes ||
      !aligned(workspace, kAlign))
    return SPARK_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* Qp = ws + L.Qp;
  void* Kp = ws + L.Kp;
  void* Vp = ws + L.Vp;
  float* qbar_blocks = reinterpret_cast<float*>(ws + L.qbar_blocks);
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  void* kt = ws + L.k_tilde;
  void* vt = ws + L.v_tilde;
  float* cbias = reinterpret_cast<float*>(ws + L.cbias);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + L.sel);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws + L.err);
  void* Kcb = ws + L.total;
  void* Vcb = ws + L.total + cbytes;

  if (cudaMemsetAsync(err, 0, sizeof(uint32_t), s) != cudaSuccess) return SPARK_ERR_CUDA;
  if (launch_gather_q(Q, dtype, H, N, d, q_perm, q_block_offsets, nqb, Qp, qbar_blocks, err, s) !=
      cudaSuccess)
    return SPARK_ERR_CUDA;
  if (launch_anchor(qbar_blocks, q_block_offsets, H, N, d, nqb, qbar, s) != cudaSuccess)
    return SPARK_ERR_CUDA;
  if (launch_gather_kv_summary(K, V, dtype, H, N, d, k_perm, k_block_offsets, nkb, qbar, Kp, Vp,
                               kbar, kt, vt, cbias, err, s) != cudaSuccess)
    return SPARK_ERR_CUDA;
  if (!fused && launch_route(qbar_blocks, kbar, H, nqb, nkb, d, L.k, sel, err, s) != cudaSuccess)
    return SPARK_ERR_CUDA;
  const void* Kca = Kc;                          // bf16 context rows are read in place
  const void* Vca = Vc;
  if (nc > 0 && dtype == SPARK_F32) {
    const size_t n = static_cast<size_t>(H) * nc * d;
    if (launch_to_bf16(Kc, dtype, n, Kcb, s) != cudaSuccess ||
        launch_to_bf16(Vc, dtype, n, Vcb, s) != cudaSuccess)
      return SPARK_ERR_CUDA;
    Kca = Kcb;
    Vca = Vcb;
  }
  if (fused)   // the selection is made inside the attention kernel and copied to the workspace
    return attend_fused_impl(Qp, Kp, Vp, kt, vt, cbias, qbar_blocks, kbar, L.k, Kca, Vca, nc,
                             q_perm, q_block_offsets, nqb, k_block_offsets, nkb, H, N, d, out,
                             dtype, err, sel, s);
  if (!fp8)
    return attend_impl(Qp, Kp, Vp, kt, vt, cbias, sel, L.k, Kca, Vca, nc, q_perm,
                       q_block_offsets, nqb, k_block_offsets, nkb, H, N, d, out, dtype, err, s);
  // FP8 logits: quantise the queries per query block, the keys per key block, the summary
  // and context keys per 128-row tile, then attend
  const Fp8Layout F = fp8_layout(H, N, d, nqb, nkb, nc);
  uint8_t* f = ws + L.total + 2 * cbytes;
  float* q_scale = reinterpret_cast<float*>(f + F.q_scale);
  float* k_scale = reinterpret_cast<float*>(f + F.k_scale);
  float* kt_scale = reinterpret_cast<float*>(f + F.kt_scale);
  float* kc_scale = reinterpret_cast<float*>(f + F.kc_scale);
  if (launch_quant_fp8(Qp, H, N, d, q_block_offsets, nqb, f + F.Qp8, q_scale, err, s) !=
          cudaSuccess ||
      launch_quant_fp8(Kp, H, N, d, k_block_offsets, nkb, f + F.Kp8, k_scale, err, s) !=
          cudaSuccess ||
      launch_quant_fp8(kt, H, nkb, d, nullptr, (nkb + 127) / 128, f + F.kt8, kt_scale, err, s) !=
          cudaSuccess)
    return SPARK_ERR_CUDA;
  if (nc > 0 && launch_quant_fp8(Kca, H, nc, d, nullptr, (nc + 127) / 128, f + F.Kc8, kc_scale,
                                 err, s) != cudaSuccess)
    return SPARK_ERR_CUDA;
  return attend_fp8_impl(f + F.Qp8, q_scale, f + F.Kp8, k_scale, Vp, f + F.kt8, kt_scale, vt,
                         cbias, sel, L.k, f + F.Kc8, kc_scale, Vca, nc, q_perm, q_block_offsets,
                         nqb, k_block_offsets, nkb, H, N, d, out, dtype, err, s);
}

}  // namespace

extern "C" {

const char* spark_status_string(int status) {
  switch (status) {
    case SPARK_OK: return "SPARK_OK";
    case SPARK_ERR_INVALID_ARG: return "SPARK_ERR_INVALID_ARG";
    case SPARK_ERR_UNSUPPORTED: return "SPARK_ERR_UNSUPPORTED";
    case SPARK_ERR_WORKSPACE: return "SPARK_ERR_WORKSPACE";
    case SPARK_ERR_CUDA: return "SPARK_ERR_CUDA";
    case SPARK_ERR_DEVICE_CHECK: return "SPARK_ERR_DEVICE_CHECK";
    default: return "SPARK_UNKNOWN_STATUS";
  }
}

int spark_bsa_topk_count(int nkb, double topk_ratio) { return topk_count(nkb, topk_ratio); }

void spark_bsa_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
}

uint64_t spark_bsa_get_wait_limit_ns(void) { return wait_limit_ns(); }

spark_status spark_bsa_workspace_layout(int H, int N, int d, int nqb, int nkb,
                                        double topk_ratio, spark_bsa_layout* layout) {
  if (layout == nullptr) return SPARK_ERR_INVALID_ARG;
  return layout_of(H, N, d, nqb, nkb, topk_ratio, layout);
}

size_t spark_bsa_workspace_size(int H, int N, int d, int nqb, int nkb, double topk_ratio) {
  spark_bsa_layout L;
  return layout_of(H, N, d, nqb, nkb, topk_ratio, &L) == SPARK_OK ? L.total : 0;
}

spark_status spark_bsa_read_error(const uint32_t* err_word, void* stream, uint32_t* flags) {
  if (err_word == nullptr || flags == nullptr) return SPARK_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, err_word, sizeof(v), cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  *flags = v;
  return v == 0 ? SPARK_OK : SPARK_ERR_DEVICE_CHECK;
}

spark_status spark_bsa_gather_q(const void* Q, int dtype, int H, int N, int d,
                                const int32_t* q_perm, const int32_t* q_block_offsets, int nqb,
                                void* Qp, float* qbar_blocks, uint32_t* err, void* stream) {
  if (!Q || !q_perm || !q_block_offsets || !Qp || !qbar_blocks) return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, 1);
  if (st != SPARK_OK) return st;
  if (!aligned(Q, 16) || !aligned(Qp, 16)) return SPARK_ERR_INVALID_ARG;
  return from_cuda(launch_gather_q(Q, dtype, H, N, d, q_perm, q_block_offsets, nqb, Qp,
                                   qbar_blocks, err, as_stream(stream)));
}

spark_status spark_bsa_anchor(const float* qbar_blocks, const int32_t* q_block_offsets, int H,
                              int N, int d, int nqb, float* qbar, void* stream) {
  if (!qbar_blocks || !q_block_offsets || !qbar) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, 1);
  if (st != SPARK_OK) return st;
  return from_cuda(launch_anchor(qbar_blocks, q_block_offsets, H, N, d, nqb, qbar,
                                 as_stream(stream)));
}

spark_status spark_bsa_gather_kv_summarize(const void* K, const void* V, int dtype, int H,
                                           int N, int d, const int32_t* k_perm,
                                           const int32_t* k_block_offsets, int nkb,
                                           const float* qbar, void* Kp, void* Vp, float* kbar,
                                           void* k_tilde, void* v_tilde, float* cbias,
                                           uint32_t* err, void* stream) {
  if (!K || !V || !k_perm || !k_block_offsets || !qbar || !Kp || !Vp || !kbar || !k_tilde ||
      !v_tilde || !cbias)
    return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, 1, nkb);
  if (st != SPARK_OK) return st;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Kp, 16) || !aligned(Vp, 16))
    return SPARK_ERR_INVALID_ARG;
  return from_cuda(launch_gather_kv_summary(K, V, dtype, H, N, d, k_perm, k_block_offsets, nkb,
                                            qbar, Kp, Vp, kbar, k_tilde, v_tilde, cbias, err,
                                            as_stream(stream)));
}

spark_status spark_bsa_gather_kv_meanpool(const void* K, const void* V, int dtype, int H, int N,
                                          int d, const int32_t* k_perm,
                                          const int32_t* k_block_offsets, int nkb, void* Kp,
                                          void* Vp, float* kbar, void* k_tilde, void* v_tilde,
                                          float* cbias, uint32_t* err, void* stream) {
  if (!K || !V || !k_perm || !k_block_offsets || !Kp || !Vp || !kbar || !k_tilde || !v_tilde ||
      !cbias)
    return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, 1, nkb);
  if (st != SPARK_OK) return st;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Kp, 16) || !aligned(Vp, 16))
    return SPARK_ERR_INVALID_ARG;
  return from_cuda(launch_gather_kv_meanpool(K, V, dtype, H, N, d, k_perm, k_block_offsets, nkb,
                                             Kp, Vp, kbar, k_tilde, v_tilde, cbias, err,
                                             as_stream(stream)));
}

spark_status spark_bsa_route(const float* qbar_blocks, const float* kbar, int H, int nqb,
                             int nkb, int d, int k, int32_t* sel, uint32_t* err, void* stream) {
  if (!qbar_blocks || !kbar || !sel) return SPARK_ERR_INVALID_ARG;
  if (H < 1 || nqb < 1 || nkb < 1 || k < 1 || k > nkb) return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (H > 65535 || nkb > kMaxNkb) return SPARK_ERR_UNSUPPORTED;
  return from_cuda(launch_route(qbar_blocks, kbar, H, nqb, nkb, d, k, sel, err,
                                as_stream(stream)));
}

spark_status spark_bsa_attend(const void* Qp, const void* Kp, const void* Vp,
                              const void* k_tilde, const void* v_tilde, const float* cbias,
                              const int32_t* sel, int k, const int32_t* q_perm,
                              const int32_t* q_block_offsets, int nqb,
                              const int32_t* k_block_offsets, int nkb, int H, int N, int d,
                              void* out, int out_dtype, uint32_t* err, void* stream) {
  if (!Qp || !Kp || !Vp || !k_tilde || !v_tilde || !cbias || !sel || !q_perm ||
      !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (out_dtype != SPARK_BF16 && out_dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  if (k < 1 || k > nkb) return SPARK_ERR_INVALID_ARG;
  if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(k_tilde, 16) ||
      !aligned(v_tilde, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  return attend_impl(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, k, nullptr, nullptr, 0, q_perm,
                     q_block_offsets, nqb, k_block_offsets, nkb, H, N, d, out, out_dtype, err,
                     as_stream(stream));
}

spark_status spark_bsa_attend_ctx(const void* Qp, const void* Kp, const void* Vp,
                                  const void* k_tilde, const void* v_tilde, const float* cbias,
                                  const int32_t* sel, int k, const void* Kc, const void* Vc,
                                  int nc, const int32_t* q_perm, const int32_t* q_block_offsets,
                                  int nqb, const int32_t* k_block_offsets, int nkb, int H, int N,
                                  int d, void* out, int out_dtype, uint32_t* err, void* stream) {
  if (!Qp || !Kp || !Vp || !k_tilde || !v_tilde || !cbias || !sel || !q_perm ||
      !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (out_dtype != SPARK_BF16 && out_dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  st = check_context(Kc, Vc, nc);
  if (st != SPARK_OK) return st;
  if (k < 1 || k > nkb) return SPARK_ERR_INVALID_ARG;
  if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(k_tilde, 16) ||
      !aligned(v_tilde, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  return attend_impl(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, k, Kc, Vc, nc, q_perm,
                     q_block_offsets, nqb, k_block_offsets, nkb, H, N, d, out, out_dtype, err,
                     as_stream(stream));
}

spark_status spark_bsa_context_bf16(const void* Kc, const void* Vc, int dtype, int H, int nc,
                                    int d, void* Kc_bf16, void* Vc_bf16, void* stream) {
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  if (H < 1 || H > 65535) return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  spark_status st = check_context(Kc, Vc, nc);
  if (st != SPARK_OK) return st;
  if (nc == 0) return SPARK_OK;
  if (!Kc_bf16 || !Vc_bf16 || !aligned(Kc_bf16, 16) || !aligned(Vc_bf16, 16))
    return SPARK_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(H) * nc * d;
  cudaStream_t s = as_stream(stream);
  if (launch_to_bf16(Kc, dtype, n, Kc_bf16, s) != cudaSuccess) return SPARK_ERR_CUDA;
  return from_cuda(launch_to_bf16(Vc, dtype, n, Vc_bf16, s));
}

size_t spark_bsa_workspace_size_ctx(int H, int N, int d, int nqb, int nkb, double topk_ratio,
                                    int nc) {
  spark_bsa_layout L;
  if (layout_of(H, N, d, nqb, nkb, topk_ratio, &L) != SPARK_OK) return 0;
  if (nc < 0 || nc > SPARK_MAX_NC) return 0;
  return L.total + (nc > 0 ? 2 * context_bytes(H, nc, d) : 0);
}

spark_status spark_bsa_forward_ctx(const void* Q, const void* K, const void* V, const void* Kc,
                                   const void* Vc, int nc, int dtype, int H, int N, int d,
                                   const int32_t* q_perm, const int32_t* k_perm,
                                   const int32_t* q_block_offsets, int nqb,
                                   const int32_t* k_block_offsets, int nkb, double topk_ratio,
                                   void* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  return forward_impl(Q, K, V, Kc, Vc, nc, dtype, H, N, d, q_perm, k_perm, q_block_offsets, nqb,
                      k_block_offsets, nkb, topk_ratio, out, workspace, workspace_bytes,
                      as_stream(stream));
}

spark_status spark_bsa_forward(const void* Q, const void* K, const void* V, int dtype, int H,
                               int N, int d, const int32_t* q_perm, const int32_t* k_perm,
                               const int32_t* q_block_offsets, int nqb,
                               const int32_t* k_block_offsets, int nkb, double topk_ratio,
                               void* out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return forward_impl(Q, K, V, nullptr, nullptr, 0, dtype, H, N, d, q_perm, k_perm,
                      q_block_offsets, nqb, k_block_offsets, nkb, topk_ratio, out, workspace,
                      workspace_bytes, as_stream(stream));
}

// ------------------------------------------------------- routing inside the attention kernel

int spark_bsa_fused_supported(int d, int nkb, double topk_ratio) {
  const int k = topk_count(nkb, topk_ratio);
  return (k >= 1 && nkb >= 1 && nkb <= kMaxNkb && attend_fused_supported(d, nkb, k)) ? 1 : 0;
}

spark_status spark_bsa_forward_fused(const void* Q, const void* K, const void* V, int dtype,
                                     int H, int N, int d, const int32_t* q_perm,
                                     const int32_t* k_perm, const int32_t* q_block_offsets,
                                     int nqb, const int32_t* k_block_offsets, int nkb,
                                     double topk_ratio, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return forward_impl(Q, K, V, nullptr, nullptr, 0, dtype, H, N, d, q_perm, k_perm,
                      q_block_offsets, nqb, k_block_offsets, nkb, topk_ratio, out, workspace,
                      workspace_bytes, as_stream(stream), false, true);
}

spark_status spark_bsa_attend_fused(const void* Qp, const void* Kp, const void* Vp,
                                    const void* k_tilde, const void* v_tilde, const float* cbias,
                                    const float* qbar_blocks, const float* kbar, int k,
                                    const int32_t* q_perm, const int32_t* q_block_offsets,
                                    int nqb, const int32_t* k_block_offsets, int nkb, int H,
                                    int N, int d, void* out, int out_dtype, int32_t* sel_out,
                                    uint32_t* err, void* stream) {
  if (!Qp || !Kp || !Vp || !k_tilde || !v_tilde || !cbias || !qbar_blocks || !kbar ||
      !q_perm || !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (out_dtype != SPARK_BF16 && out_dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  if (k < 1 || k > nkb) return SPARK_ERR_INVALID_ARG;
  if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(k_tilde, 16) ||
      !aligned(v_tilde, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  return attend_fused_impl(Qp, Kp, Vp, k_tilde, v_tilde, cbias, qbar_blocks, kbar, k, nullptr,
                           nullptr, 0, q_perm, q_block_offsets, nqb, k_block_offsets, nkb, H, N,
                           d, out, out_dtype, err, sel_out, as_stream(stream));
}

// ----------------------------------------------------------- threshold routing (comparator)

spark_status spark_bsa_route_threshold(const float* qbar_blocks, const float* kbar, int H,
                                       int nqb, int nkb, int d, double tau, int kcap,
                                       int32_t* sel, int32_t* count, uint32_t* err,
                                       void* stream) {
  if (!qbar_blocks || !kbar || !sel || !count) return SPARK_ERR_INVALID_ARG;
  if (H < 1 || nqb < 1 || nkb < 1 || kcap < 1 || kcap > nkb || !(tau == tau))
    return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (H > 65535 || nkb > kMaxNkb) return SPARK_ERR_UNSUPPORTED;
  (void)err;
  return from_cuda(launch_route_threshold(qbar_blocks, kbar, H, nqb, nkb, d,
                                          static_cast<float>(tau), kcap, sel, count,
                                          as_stream(stream)));
}

spark_status spark_bsa_attend_var(const void* Qp, const void* Kp, const void* Vp,
                                  const void* k_tilde, const void* v_tilde, const float* cbias,
                                  const int32_t* sel, int kcap, const int32_t* count,
                                  const int32_t* q_perm, const int32_t* q_block_offsets, int nqb,
                                  const int32_t* k_block_offsets, int nkb, int H, int N, int d,
                                  void* out, int out_dtype, uint32_t* err, void* stream) {
  if (!Qp || !Kp || !Vp || !k_tilde || !v_tilde || !cbias || !sel || !count || !q_perm ||
      !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (out_dtype != SPARK_BF16 && out_dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  if (kcap < 1 || kcap > nkb) return SPARK_ERR_INVALID_ARG;
  if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(k_tilde, 16) ||
      !aligned(v_tilde, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  return attend_impl(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, kcap, nullptr, nullptr, 0, q_perm,
                     q_block_offsets, nqb, k_block_offsets, nkb, H, N, d, out, out_dtype, err,
                     as_stream(stream), count);
}

// ------------------------------------------------------------------------ FP8 logits

spark_status spark_bsa_quantize_fp8(const void* src, int H, int R, int d,
                                    const int32_t* group_offsets, int ngroups, void* dst,
                                    float* scales, uint32_t* err, void* stream) {
  if (!src || !dst || !scales) return SPARK_ERR_INVALID_ARG;
  if (H < 1 || H > 65535 || R < 1 || ngroups < 1) return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (group_offsets == nullptr && ngroups != (R + 127) / 128) return SPARK_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16)) return SPARK_ERR_INVALID_ARG;
  return from_cuda(launch_quant_fp8(src, H, R, d, group_offsets, ngroups, dst, scales, err,
                                    as_stream(stream)));
}

spark_status spark_bsa_attend_fp8(const void* Qp8, const float* q_scale, const void* Kp8,
                                  const float* k_scale, const void* Vp, const void* kt8,
                                  const float* kt_scale, const void* v_tilde,
                                  const float* cbias, const int32_t* sel, int k,
                                  const void* Kc8, const float* kc_scale, const void* Vc, int nc,
                                  const int32_t* q_perm, const int32_t* q_block_offsets,
                                  int nqb, const int32_t* k_block_offsets, int nkb, int H,
                                  int N, int d, void* out, int out_dtype, uint32_t* err,
                                  void* stream) {
  if (!Qp8 || !q_scale || !Kp8 || !k_scale || !Vp || !kt8 || !kt_scale || !v_tilde || !cbias ||
      !sel || !q_perm || !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (out_dtype != SPARK_BF16 && out_dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_status st = check_sizes(H, N, d, nqb, nkb);
  if (st != SPARK_OK) return st;
  if (d != 128) return SPARK_ERR_UNSUPPORTED;
  st = check_context(Kc8, Vc, nc);
  if (st != SPARK_OK) return st;
  if (nc > 0 && !kc_scale) return SPARK_ERR_INVALID_ARG;
  if (k < 1 || k > nkb) return SPARK_ERR_INVALID_ARG;
  if (!aligned(Qp8, 16) || !aligned(Kp8, 16) || !aligned(Vp, 16) || !aligned(kt8, 16) ||
      !aligned(v_tilde, 16) || !aligned(out, 16))
    return SPARK_ERR_INVALID_ARG;
  return attend_fp8_impl(Qp8, q_scale, Kp8, k_scale, Vp, kt8, kt_scale, v_tilde, cbias, sel, k,
                         Kc8, kc_scale, Vc, nc, q_perm, q_block_offsets, nqb, k_block_offsets,
                         nkb, H, N, d, out, out_dtype, err, as_stream(stream));
}

size_t spark_bsa_workspace_size_fp8(int H, int N, int d, int nqb, int nkb, double topk_ratio,
                                    int nc) {
  if (d != 128) return 0;
  const size_t base = spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, topk_ratio, nc);
  if (base == 0) return 0;
  return base + fp8_layout(H, N, d, nqb, nkb, nc).total;
}

spark_status spark_bsa_forward_fp8(const void* Q, const void* K, const void* V, const void* Kc,
                                   const void* Vc, int nc, int dtype, int H, int N, int d,
                                   const int32_t* q_perm, const int32_t* k_perm,
                                   const int32_t* q_block_offsets, int nqb,
                                   const int32_t* k_block_offsets, int nkb, double topk_ratio,
                                   void* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  return forward_impl(Q, K, V, Kc, Vc, nc, dtype, H, N, d, q_perm, k_perm, q_block_offsets, nqb,
                      k_block_offsets, nkb, topk_ratio, out, workspace, workspace_bytes,
                      as_stream(stream), true);
}

// ------------------------------------------------- host buffers, pipelined by head chunks

namespace {

struct HostStaging {
  size_t Q, K, V, qp, kp, out, Kc, Vc, slot, qo, ko, total;
};

HostStaging staging_layout(int hpc, int N, int d, int esize, int nqb, int nkb, int nc = 0) {
  HostStaging L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t rows = static_cast<size_t>(hpc) * N;
  L.Q = take(rows * d * esize);
  L.K = take(rows * d * esize);
  L.V = take(rows * d * esize);
  L.qp = take(rows * 4);
  L.kp = take(rows * 4);
  L.out = take(rows * d * esize);
  L.Kc = take(static_cast<size_t>(hpc) * nc * d * esize);   // context rows of the chunk's heads
  L.Vc = take(static_cast<size_t>(hpc) * nc * d * esize);
  L.slot = off;                                  // one slot; the second follows at +slot
  off = 2 * L.slot;
  L.qo = take(static_cast<size_t>(nqb + 1) * 4);
  L.ko = take(static_cast<size_t>(nkb + 1) * 4);
  L.total = off;
  return L;
}

}  // namespace

size_t spark_bsa_host_staging_size(int H, int N, int d, int dtype, int nqb, int nkb,
                                   int heads_per_chunk) {
  if (check_sizes(H, N, d, nqb, nkb) != SPARK_OK || heads_per_chunk < 1) return 0;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return 0;
  const int hpc = heads_per_chunk < H ? heads_per_chunk : H;
  return staging_layout(hpc, N, d, dtype == SPARK_BF16 ? 2 : 4, nqb, nkb).total;
}

namespace {

// The host-buffer pipeline for every variant: nc context rows per head (Kc, Vc host [H,nc,d],
// none when nc == 0) and FP8 logits when fp8 is set.
spark_status forward_host_impl(const void* Q, const void* K, const void* V, const void* Kc,
                               const void* Vc, int nc, bool fp8, int dtype, int H, int N, int d,
                               const int32_t* q_perm, const int32_t* k_perm,
                               const int32_t* q_block_offsets, int nqb,
                               const int32_t* k_block_offsets, int nkb, double topk_ratio,
                               void* out, int heads_per_chunk, void* staging,
                               size_t staging_bytes, void* workspace, size_t workspace_bytes,
                               void* compute_stream, void* h2d_stream, void* d2h_stream) {
  if (!Q || !K || !V || !q_perm || !k_perm || !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  if (heads_per_chunk < 1) return SPARK_ERR_INVALID_ARG;
  if (nc < 0 || nc > SPARK_MAX_NC || (nc > 0 && (!Kc || !Vc))) return SPARK_ERR_INVALID_ARG;
  if (fp8 && d != 128) return SPARK_ERR_UNSUPPORTED;
  spark_bsa_layout whole;
  spark_status st = layout_of(H, N, d, nqb, nkb, topk_ratio, &whole);
  if (st != SPARK_OK) return st;
  const int hpc = heads_per_chunk < H ? heads_per_chunk : H;
  const size_t chunk_ws = fp8 ? spark_bsa_workspace_size_fp8(hpc, N, d, nqb, nkb, topk_ratio, nc)
                              : spark_bsa_workspace_size_ctx(hpc, N, d, nqb, nkb, topk_ratio, nc);
  if (chunk_ws == 0) return SPARK_ERR_INVALID_ARG;
  const int esize = dtype == SPARK_BF16 ? 2 : 4;
  const HostStaging S = staging_layout(hpc, N, d, esize, nqb, nkb, nc);
  if (!staging || staging_bytes < S.total || !aligned(staging, kAlign)) return SPARK_ERR_WORKSPACE;
  if (!workspace || workspace_bytes < chunk_ws || !aligned(workspace, kAlign))
    return SPARK_ERR_WORKSPACE;
  cudaStream_t sc = as_stream(compute_stream), sh = as_stream(h2d_stream),
               sd = as_stream(d2h_stream);
  uint8_t* stg = static_cast<uint8_t*>(staging);
  cudaEvent_t ev[7] = {};
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (auto& f : ev)
        if (f) cudaEventDestroy(f);
      return SPARK_ERR_CUDA;
    }
  cudaEvent_t* h2d_done = ev;        // [2]
  cudaEvent_t* comp_done = ev + 2;   // [2]
  cudaEvent_t* d2h_done = ev + 4;    // [2]
  cudaEvent_t start = ev[6];
  auto fail = [&]() {
    for (auto& e : ev) cudaEventDestroy(e);
    return SPARK_ERR_CUDA;
  };
  // the copy streams start after everything already queued on the compute stream (e.g. an
  // earlier call that still reads the staging slots)
  if (cudaEventRecord(start, sc) != cudaSuccess || cudaStreamWaitEvent(sh, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(sd, start, 0) != cudaSuccess)
    return fail();
  const size_t row_bytes = static_cast<size_t>(N) * d * esize;
  const size_t perm_bytes = static_cast<size_t>(N) * 4;
  int32_t* qo = reinterpret_cast<int32_t*>(stg + S.qo);
  int32_t* ko = reinterpret_cast<int32_t*>(stg + S.ko);
  if (cudaMemcpyAsync(qo, q_block_offsets, (nqb + 1) * 4, cudaMemcpyHostToDevice, sh) !=
          cudaSuccess ||
      cudaMemcpyAsync(ko, k_block_offsets, (nkb + 1) * 4, cudaMemcpyHostToDevice, sh) !=
          cudaSuccess)
    return fail();
  const int nchunks = (H + hpc - 1) / hpc;
  const auto* q8 = static_cast<const uint8_t*>(Q);
  const auto* k8 = static_cast<const uint8_t*>(K);
  const auto* v8 = static_cast<const uint8_t*>(V);
  const auto* kc8 = static_cast<const uint8_t*>(Kc);
  const auto* vc8 = static_cast<const uint8_t*>(Vc);
  const size_t ctx_bytes = static_cast<size_t>(nc) * d * esize;   // one head's context rows
  auto* o8 = static_cast<uint8_t*>(out);
  for (int c = 0; c < nchunks; ++c) {
    const int slot = c & 1;
    const int h0 = c * hpc;
    const int hc = (H - h0) < hpc ? (H - h0) : hpc;
    uint8_t* base = stg + slot * S.slot;
    // inputs of chunk c into the slot, once chunk c-2 no longer reads it
    if (c >= 2 && cudaStreamWaitEvent(sh, comp_done[slot], 0) != cudaSuccess) return fail();
    if (cudaMemcpyAsync(base + S.Q, q8 + h0 * row_bytes, hc * row_bytes, cudaMemcpyHostToDevice,
                        sh) != cudaSuccess ||
        cudaMemcpyAsync(base + S.K, k8 + h0 * row_bytes, hc * row_bytes, cudaMemcpyHostToDevice,
                        sh) != cudaSuccess ||
        cudaMemcpyAsync(base + S.V, v8 + h0 * row_bytes, hc * row_bytes, cudaMemcpyHostToDevice,
                        sh) != cudaSuccess ||
        cudaMemcpyAsync(base + S.qp, q_perm + static_cast<size_t>(h0) * N, hc * perm_bytes,
                        cudaMemcpyHostToDevice, sh) != cudaSuccess ||
        cudaMemcpyAsync(base + S.kp, k_perm + static_cast<size_t>(h0) * N, hc * perm_bytes,
                        cudaMemcpyHostToDevice, sh) != cudaSuccess)
      return fail();
    if (nc > 0 &&
        (cudaMemcpyAsync(base + S.Kc, kc8 + h0 * ctx_bytes, hc * ctx_bytes,
                         cudaMemcpyHostToDevice, sh) != cudaSuccess ||
         cudaMemcpyAsync(base + S.Vc, vc8 + h0 * ctx_bytes, hc * ctx_bytes,
                         cudaMemcpyHostToDevice, sh) != cudaSuccess))
      return fail();
    if (cudaEventRecord(h2d_done[slot], sh) != cudaSuccess) return fail();
    // the forward pass of the chunk, once its inputs are in and the slot's output is read out
    if (cudaStreamWaitEvent(sc, h2d_done[slot], 0) != cudaSuccess) return fail();
    if (c >= 2 && cudaStreamWaitEvent(sc, d2h_done[slot], 0) != cudaSuccess) return fail();
    st = forward_impl(base + S.Q, base + S.K, base + S.V, nc > 0 ? base + S.Kc : nullptr,
                      nc > 0 ? base + S.Vc : nullptr, nc, dtype, hc, N, d,
                      reinterpret_cast<const int32_t*>(base + S.qp),
                      reinterpret_cast<const int32_t*>(base + S.kp), qo, nqb, ko, nkb,
                      topk_ratio, base + S.out, workspace, workspace_bytes, sc, fp8);
    if (st != SPARK_OK) {
      for (auto& e : ev) cudaEventDestroy(e);
      return st;
    }
    if (cudaEventRecord(comp_done[slot], sc) != cudaSuccess) return fail();
    // the chunk's output back to the host
    if (cudaStreamWaitEvent(sd, comp_done[slot], 0) != cudaSuccess ||
        cudaMemcpyAsync(o8 + h0 * row_bytes, base + S.out, hc * row_bytes,
                        cudaMemcpyDeviceToHost, sd) != cudaSuccess ||
        cudaEventRecord(d2h_done[slot], sd) != cudaSuccess)
      return fail();
  }
  // the compute stream completes only after every copy back
  for (int slot = 0; slot < 2 && slot < nchunks; ++slot)
    if (cudaStreamWaitEvent(sc, d2h_done[slot], 0) != cudaSuccess) return fail();
  for (auto& e : ev) cudaEventDestroy(e);   // released once the pending work completes
  return SPARK_OK;
}

}  // namespace

spark_status spark_bsa_forward_host(const void* Q, const void* K, const void* V, int dtype,
                                    int H, int N, int d, const int32_t* q_perm,
                                    const int32_t* k_perm, const int32_t* q_block_offsets,
                                    int nqb, const int32_t* k_block_offsets, int nkb,
                                    double topk_ratio, void* out, int heads_per_chunk,
                                    void* staging, size_t staging_bytes, void* workspace,
                                    size_t workspace_bytes, void* compute_stream,
                                    void* h2d_stream, void* d2h_stream) {
  return forward_host_impl(Q, K, V, nullptr, nullptr, 0, false, dtype, H, N, d, q_perm, k_perm,
                           q_block_offsets, nqb, k_block_offsets, nkb, topk_ratio, out,
                           heads_per_chunk, staging, staging_bytes, workspace, workspace_bytes,
                           compute_stream, h2d_stream, d2h_stream);
}

size_t spark_bsa_host_staging_size_ex(int H, int N, int d, int dtype, int nqb, int nkb,
                                      int heads_per_chunk, int nc) {
  if (check_sizes(H, N, d, nqb, nkb) != SPARK_OK || heads_per_chunk < 1) return 0;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return 0;
  if (nc < 0 || nc > SPARK_MAX_NC) return 0;
  const int hpc = heads_per_chunk < H ? heads_per_chunk : H;
  return staging_layout(hpc, N, d, dtype == SPARK_BF16 ? 2 : 4, nqb, nkb, nc).total;
}

spark_status spark_bsa_forward_host_ex(const void* Q, const void* K, const void* V,
                                       const void* Kc, const void* Vc, int nc, int fp8_logits,
                                       int dtype, int H, int N, int d, const int32_t* q_perm,
                                       const int32_t* k_perm, const int32_t* q_block_offsets,
                                       int nqb, const int32_t* k_block_offsets, int nkb,
                                       double topk_ratio, void* out, int heads_per_chunk,
                                       void* staging, size_t staging_bytes, void* workspace,
                                       size_t workspace_bytes, void* compute_stream,
                                       void* h2d_stream, void* d2h_stream) {
  return forward_host_impl(Q, K, V, Kc, Vc, nc, fp8_logits != 0, dtype, H, N, d, q_perm, k_perm,
                           q_block_offsets, nqb, k_block_offsets, nkb, topk_ratio, out,
                           heads_per_chunk, staging, staging_bytes, workspace, workspace_bytes,
                           compute_stream, h2d_stream, d2h_stream);
}

// ---------------------------------------------------------------- Spark-Reblock

int spark_reblock_levels(int N, int block) {
  if (N < 1 || block < 1 || block > SPARK_MAX_BLOCK) return -1;
  return static_cast<int>(reblock_levels(N, block));
}

spark_status spark_reblock_workspace_layout(int H, int N, int d, int block,
                                            spark_reblock_layout* layout) {
  if (layout == nullptr || H < 1 || N < 1 || block < 1 || block > SPARK_MAX_BLOCK)
    return SPARK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARK_ERR_UNSUPPORTED;
  if (H > 65535 || (N + block - 1) / block > kMaxNkb) return SPARK_ERR_UNSUPPORTED;
  const ReblockLayout L = reblock_layout(H, N, d, block);
  layout->M = L.M;
  layout->W = L.W;
  layout->X = L.X;
  layout->total = L.total;
  layout->levels = L.levels;
  layout->nb = L.nb;
  return SPARK_OK;
}

size_t spark_reblock_workspace_size(int H, int N, int d, int block) {
  spark_reblock_layout L;
  return spark_reblock_workspace_layout(H, N, d, block, &L) == SPARK_OK ? L.total : 0;
}

spark_status spark_reblock_whiten(const void* X, const void* Y, int dtype, int H, int N, int d,
                                  int block, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!X || !Y) return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  spark_reblock_layout pub;
  spark_status st = spark_reblock_workspace_layout(H, N, d, block, &pub);
  if (st != SPARK_OK) return st;
  if (!aligned(X, 16) || !aligned(Y, 16)) return SPARK_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pub.total || !aligned(workspace, kAlign))
    return SPARK_ERR_WORKSPACE;
  const ReblockLayout L = reblock_layout(H, N, d, block);
  return from_cuda(launch_reblock_whiten(X, Y, dtype, H, N, d, workspace, L, as_stream(stream)));
}

spark_status spark_reblock_level(int H, int N, int d, int block, int level,
                                 const int32_t* perm_in, int32_t* perm_out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!perm_in || !perm_out || perm_in == perm_out) return SPARK_ERR_INVALID_ARG;
  spark_reblock_layout pub;
  spark_status st = spark_reblock_workspace_layout(H, N, d, block, &pub);
  if (st != SPARK_OK) return st;
  if (level < 0 || level >= pub.levels) return SPARK_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pub.total || !aligned(workspace, kAlign))
    return SPARK_ERR_WORKSPACE;
  const ReblockLayout L = reblock_layout(H, N, d, block);
  cudaStream_t s = as_stream(stream);
  if (upload_reblock_plan(N, block, workspace, L, s) != cudaSuccess) return SPARK_ERR_CUDA;
  return from_cuda(launch_reblock_level(H, N, d, block, level, perm_in, perm_out, workspace, L, s));
}

spark_status spark_reblock(const void* Q, const void* K, int dtype, int H, int N, int d,
                           int block, int mode, int32_t* q_perm, int32_t* k_perm,
                           int32_t* offsets, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!Q || !K || !q_perm || !k_perm || !offsets) return SPARK_ERR_INVALID_ARG;
  if (dtype != SPARK_BF16 && dtype != SPARK_F32) return SPARK_ERR_INVALID_ARG;
  if (mode != SPARK_REBLOCK_Q_REUSE_K && mode != SPARK_REBLOCK_SEPARATE)
    return SPARK_ERR_INVALID_ARG;
  spark_reblock_layout pub;
  spark_status st = spark_reblock_workspace_layout(H, N, d, block, &pub);
  if (st != SPARK_OK) return st;
  if (!aligned(Q, 16) || !aligned(K, 16)) return SPARK_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pub.total || !aligned(workspace, kAlign))
    return SPARK_ERR_WORKSPACE;
  const ReblockLayout L = reblock_layout(H, N, d, block);
  cudaStream_t s = as_stream(stream);
  if (launch_reblock_whiten(Q, K, dtype, H, N, d, workspace, L, s) != cudaSuccess ||
      launch_reblock_partition(H, N, d, block, q_perm, workspace, L, s) != cudaSuccess)
    return SPARK_ERR_CUDA;
  if (mode == SPARK_REBLOCK_SEPARATE) {
    if (launch_reblock_whiten(K, Q, dtype, H, N, d, workspace, L, s) != cudaSuccess ||
        launch_reblock_partition(H, N, d, block, k_perm, workspace, L, s) != cudaSuccess)
      return SPARK_ERR_CUDA;
  } else if (cudaMemcpyAsync(k_perm, q_perm, static_cast<size_t>(H) * N * 4,
                             cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    return SPARK_ERR_CUDA;
  }
  return from_cuda(launch_reblock_offsets(offsets, L.nb, N, block, s));
}

}  // extern "C"
