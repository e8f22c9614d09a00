// Kernel launchers shared by the C ABI (api.cu) and the kernel files.
#pragma once

#include "spark_ptx.cuh"

namespace spark {

constexpr int kMaxBlock = 128;     // tokens per block (one MMA tile of keys / queries)
constexpr int kMaxNkb = 12800;     // key blocks per head accepted by the routing kernel

// Limit of every bounded wait in the kernels launched from now on (nanoseconds): the
// process-wide setting of spark_bsa_set_wait_limit_ns, kWaitLimitNs by default (api.cu).
uint64_t wait_limit_ns();

cudaError_t launch_gather_q(const void* Q, int dtype, int H, int N, int d,
                            const int32_t* q_perm, const int32_t* q_offsets, int nqb, void* Qp,
                            float* qbar_blocks, uint32_t* err, cudaStream_t s);

cudaError_t launch_anchor(const float* qbar_blocks, const int32_t* q_offsets, int H, int N,
                          int d, int nqb, float* qbar, cudaStream_t s);

cudaError_t launch_gather_kv_summary(const void* K, const void* V, int dtype, int H, int N,
                                     int d, const int32_t* k_perm, const int32_t* k_offsets,
                                     int nkb, const float* qbar, void* Kp, void* Vp,
                                     float* kbar, void* k_tilde, void* v_tilde, float* cbias,
                                     uint32_t* err, cudaStream_t s);

// The baseline BSA compressed branch (mean key, mean value, offset log|B|) with the same
// gather and key-block means as launch_gather_kv_summary.
cudaError_t launch_gather_kv_meanpool(const void* K, const void* V, int dtype, int H, int N,
                                      int d, const int32_t* k_perm, const int32_t* k_offsets,
                                      int nkb, void* Kp, void* Vp, float* kbar, void* k_tilde,
                                      void* v_tilde, float* cbias, uint32_t* err,
                                      cudaStream_t s);

cudaError_t launch_route(const float* qbar_blocks, const float* kbar, int H, int nqb, int nkb,
                         int d, int k, int32_t* sel, uint32_t* err, cudaStream_t s);

// Threshold routing: per (h, A) the blocks scoring above mu + tau*sigma of the row (at most
// kcap, the largest), written ascending to the first count[h, A] entries of sel's row.
cudaError_t launch_route_threshold(const float* qbar_blocks, const float* kbar, int H, int nqb,
                                   int nkb, int d, float tau, int kcap, int32_t* sel,
                                   int32_t* count, cudaStream_t s);

// Context rows converted to bf16: dst[i] = bf16(src[i]) for n elements (a plain copy for
// bf16 sources).
cudaError_t launch_to_bf16(const void* src, int dtype, size_t n, void* dst, cudaStream_t s);

// Operands of the attention kernel: TMA descriptors (encoded on the host by api.cu) of the
// reblocked Q, K, V ([H,N,d] bf16), of the summaries k~, v~ ([H,nkb,d] bf16) and of the
// context rows Kc, Vc ([H,nc,d] bf16; unused when nc == 0).
struct AttendMaps {
  CUtensorMap q, k, v, kt, vt, kc, vc;
};

// sel rows are k apart; sel_count (optional [H,nqb]) gives each query block its own number
// of selected blocks (<= k), as threshold routing produces.
cudaError_t launch_attend(const AttendMaps& maps, int nc, const float* cbias,
                          const int32_t* sel, int k, const int32_t* q_perm,
                          const int32_t* q_offsets, int nqb, const int32_t* k_offsets, int nkb,
                          int H, int N, int d, void* out, int out_dtype, uint32_t* err,
                          cudaStream_t s, const int32_t* sel_count = nullptr);

// The attention with the routing inside (d = 128, bf16, Top-K): one persistent CTA per SM
// walks the query blocks head-major; its K producer scores and selects the next query block
// (from qbar_blocks [H,nqb,d] and kbar [H,d,nkb], the routing kernel's arithmetic) while the
// current one is attended.  sel_out (optional [H,nqb,k]) receives a copy of every selection.
bool attend_fused_supported(int d, int nkb, int k);
cudaError_t launch_attend_fused(const AttendMaps& maps, int nc, const float* cbias,
                                const float* qbar_blocks, const float* kbar, int k,
                                const int32_t* q_perm, const int32_t* q_offsets, int nqb,
                                const int32_t* k_offsets, int nkb, int H, int N, int d, void* out,
                                int out_dtype, uint32_t* err, int32_t* sel_out, cudaStream_t s);

// 3-D bf16 tensor map [H][rows][d], box 64 columns x 128 rows, 128-byte swizzle (api.cu).
bool encode_rows_map(CUtensorMap* m, const void* base, int H, int rows, int d);
// 3-D e4m3 (byte) tensor map [H][rows][d], box 128 bytes x 128 rows, 128-byte swizzle.
bool encode_rows_map_u8(CUtensorMap* m, const void* base, int H, int rows, int d);

// FP8 logits: the attention with e4m3 Q, K, k~, Kc operands (maps from encode_rows_map_u8)
// and their group scales, bf16 V, v~, Vc (d = 128).
cudaError_t launch_attend_fp8(const AttendMaps& maps, const float* q_scale,
                              const float* k_scale, const float* kt_scale,
                              const float* kc_scale, int nc, const float* cbias,
                              const int32_t* sel, int k, const int32_t* q_perm,
                              const int32_t* q_offsets, int nqb, const int32_t* k_offsets,
                              int nkb, int H, int N, void* out, int out_dtype, uint32_t* err,
                              cudaStream_t s);

// e4m3 codes of bf16 rows [H,R,d], one power-of-two scale per group: the blocks of `offsets`
// ([ngroups+1], shared by all heads), or 128-row tiles when offsets is null (quant.cu).
cudaError_t launch_quant_fp8(const void* src, int H, int R, int d, const int32_t* offsets,
                             int ngroups, void* dst, float* scales, uint32_t* err,
                             cudaStream_t s);

// ---- Spark-Reblock partitioner (reblock.cu)
// Byte offsets of its workspace regions (256-byte aligned).
struct ReblockLayout {
  size_t mpart, M, W, Wb, X, perm0, perm1, keys, meta, part, cpart, mu, v, hist, state, cnt, base,
      err, total;
  int levels, nb;
};

ReblockLayout reblock_layout(int H, int N, int d, int block);
size_t reblock_levels(int N, int block);

// M = second moment of Yin's rows, W = M^{1/2}, workspace X = bf16 unit rows of W Xin.
cudaError_t launch_reblock_whiten(const void* Xin, const void* Yin, int dtype, int H, int N,
                                  int d, void* workspace, const ReblockLayout& L,
                                  cudaStream_t s);
// Copies the block tree's node / chunk tables into the workspace.
cudaError_t upload_reblock_plan(int N, int block, void* workspace, const ReblockLayout& L,
                                cudaStream_t s);
// One level of splits of the workspace's X rows: perm_in -> perm_out ([H,N] positions).
cudaError_t launch_reblock_level(int H, int N, int d, int block, int level,
                                 const int32_t* perm_in, int32_t* perm_out, void* workspace,
                                 const ReblockLayout& L, cudaStream_t s);
// All levels from the identity order; the final permutation goes to perm_out.
cudaError_t launch_reblock_partition(int H, int N, int d, int block, int32_t* perm_out,
                                     void* workspace, const ReblockLayout& L, cudaStream_t s);
cudaError_t launch_reblock_offsets(int32_t* offsets, int nb, int N, int block, cudaStream_t s);

}  // namespace spark
