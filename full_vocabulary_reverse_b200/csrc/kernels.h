// kernels.h -- launcher interface between the C-ABI layer (api.cu) and the
// kernel translation units.  Host-only declarations; no torch types.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace rkl {

// Kernel ids for the measurement hooks (rkl_profile_*).
enum KernelId : int {
  K_COMPACT = 0,
  K_GATHER,
  K_FWD_DUAL_TC,      // S3 hidden payload, tcgen05 (z_s and z_t, online stats)
  K_FWD_SINGLE_TC,    // S3 logits payload, tcgen05 (z_s, teacher rows loaded)
  K_TEACHER_LSE,      // S8 teacher log-sum-exp, bandwidth bound
  K_COMBINE,          // S4 merge split statistics
  K_SCATTER_LOSS,     // S4 loss_tok scatter
  K_REDUCE,           // S4 scalar loss
  K_ROW_WEIGHTS,      // S5
  K_DZ_DUAL_TC,       // S6 hidden payload, tcgen05 recompute + dz
  K_DZ_SINGLE_TC,     // S6 logits payload
  K_GRAD_TC,          // S7 dW_s and dH_s tiles (grouped), tcgen05
  K_SCATTER_DH,       // S7 dH scatter to [T, H]
  K_FWD_SIMT,         // fp32 S3 (CUDA cores)
  K_DZ_SIMT,          // fp32 S6
  K_GRAD_SIMT,        // fp32 S7
  K_PAIR_FWD,         // both sides as logits: forward statistics, bandwidth bound
  K_PAIR_BWD,         // both sides as logits: dL/dz_s rows, bandwidth bound
  K_COUNT_TEACHERS,   // per-row teachers: trainable rows per teacher
  K_BUILD_SLOTS,      // per-row teachers: teacher-grouped row slots
  K_TOPK_FWD,         // top-k estimator, both sides as logits: selection + estimate
  K_TOPK_BWD,         // top-k estimator: gradient estimate rows
  K_ZW_DUAL_TC,       // top-k, hidden payload: z_s and z_t of a row block written by tcgen05
  K_DZ_TOPK_TC,       // top-k, hidden payload: recompute + top-k dz chunk
  K_TOPK_ROWK,        // top-k, hidden payload: per-row constants of the dz pass
  K_ZW_SINGLE_TC,     // top-k, logits payload: z_s of a row block by tcgen05, shipped z_t copied beside it
  K_DZ_TOPK_SINGLE_TC,  // top-k, logits payload: recompute z_s + top-k dz chunk
  K_COUNT
};

const char* kernel_name(int id);

// Device error word bits (reported by rkl_device_error).
enum : int {
  ERR_WAIT_TMA_EMPTY = 1 << 0,   // producer waited too long for a free smem stage
  ERR_WAIT_TMA_FULL = 1 << 1,    // MMA issuer waited too long for operands
  ERR_WAIT_ACC_EMPTY = 1 << 2,   // MMA issuer waited too long for a free accumulator
  ERR_WAIT_ACC_FULL = 1 << 3,    // epilogue waited too long for an accumulator
  ERR_WAIT_AUX = 1 << 4,         // epilogue waited too long for an auxiliary tile
  ERR_WAIT_TEARDOWN = 1 << 5,    // teardown wait for in-flight MMAs ran out
  ERR_BOUNDS = 1 << 6,           // a bounds check of the RKL_DEBUG build failed
};

// Records (optionally timed) launches; implemented in api.cu.
struct LaunchScope {
  LaunchScope(int id, cudaStream_t s);
  ~LaunchScope();
  int id;
  cudaStream_t stream;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
};

// Trainable-row counts.  Every launcher takes the count as `n` (host) and an
// optional device pointer `n_dev`.  Without n_dev, n is the exact count.
// With n_dev, n is an upper bound (grids, tensor maps and workspace regions
// are sized for it) and the kernels read the live count from *n_dev at run
// time, clamped to [0, n], so that a step needs no host read of the count.
#ifdef __CUDACC__
__device__ __forceinline__ int live_rows(const int32_t* n_dev, int cap, int base = 0) {
  if (n_dev == nullptr) return cap;
  const int n = *n_dev - base;
  return n < 0 ? 0 : (n > cap ? cap : n);
}
#endif

constexpr int kBM = 128;       // rows per tile (TMEM lanes)
constexpr int kFBN = 256;      // vocab columns per fused pair tile
constexpr int kBK = 64;        // K per pipeline stage (128 B of bf16)
constexpr int kGradBN = 512;   // H columns per gradient pair tile (two N = 256 halves)
constexpr int kGroupTiles = 4;  // 256-column vocab tiles per forward statistics group (1024 columns)
// Epilogue warps of the forward statistics kernel with ng GEMMs (a multiple
// of 4: each TMEM lane quarter is read by fwd_epi / 4 warps, each owning
// 256 / (fwd_epi / 4) columns of the tile) and its statistics slots per
// vocab group.  The hidden payload (ng = 2) drains each tile with 16 warps,
// so that a warp holds two 32-column chunks and the accumulator is released
// to the next tile after one chunk of statistics work; the logits payload
// (ng = 1) keeps 8, whose registers also carry the prefetched teacher rows.
__host__ __device__ constexpr int fwd_epi(int ng) { return ng == 2 ? 16 : 8; }
__host__ __device__ constexpr int fwd_slots(int ng) { return fwd_epi(ng) / 4; }
constexpr int kStatVals = 6;    // per slot: m_s, S_s, A, m_t, S_t, sum e^(z_s-m_s) z_s
constexpr int kMaxTeachers = 16;  // teacher heads of the per-row-teacher mode

// ---------------------------------------------------------------- tcgen05
struct FusedArgs {
  // operand maps (bf16, 128-byte swizzle): A box {64, 128}, B box {64, 128}
  CUtensorMap tm_as, tm_at, tm_bs, tm_bt;
  CUtensorMap tm_dz;                 // dz chunk output [N, cw] bf16, box {64, 32}
  const uint16_t* teacher;           // logits payload: teacher logits [T, V] bf16
  const int32_t* teacher_rows;       // logits payload: row_idx (nullptr = identity)
  long long teacher_pitch;           // elements per teacher row
  float* part;                       // stats: [2G][kStatVals][n_pad]
  const float* rowc;                 // dz: [3][n_pad]: lse_s*log2e, cst, g
  const int32_t* row_idx;            // stats: compacted row -> token position
  const int32_t* targets;            // stats: target token id per position (nullable)
  float* tlogit;                     // stats: z_s at the target column [n_pad]
  int N, n_pad, H, V, KB;
  const int32_t* n_dev;              // live row count on the device (nullable: N exact)
  int n_base;                        // first compacted row of this launch (count offset)
  int IT;                            // 256-column vocab tiles per row tile in this launch
  int vt_base;                       // first 256-column vocab tile of this launch
  int GT;                            // vocab tiles per unit (group)
  int G;                             // units per m-tile = ceil(IT / GT)
  int chunk_v0;                      // dz: first vocab column of the chunk
  // Teacher per row: tm_bt covers the stacked heads [tgroups * V, H] and the
  // rows of teacher g occupy [group_row_end[g-1], group_row_end[g]) (whole
  // 256-row pair tiles).  tgroups <= 1: one teacher head.
  int tgroups;
  int group_row_end[kMaxTeachers];
  // Top-k estimator on the hidden payload.  Logit writer: z_s, z_t fp32
  // [rows, V] outputs (box {32, 32}).  Top-k dz: per-row constants
  // rowk [6][n_pad] = (lse_t - lse_s, C, a, bits of K*, bits of v_last,
  // bits of the sampled token id).
  CUtensorMap tm_zs, tm_zt;
  const float* rowk;
};

struct GradArgs {
  CUtensorMap tm_dz_k;    // dz chunk [N, cw] bf16 as K-major A (box {64, 128})
  CUtensorMap tm_dz_mn;   // dz chunk as MN-major A (box {64, 64})
  CUtensorMap tm_hs_mn;   // hc_s [N, H] bf16 as MN-major B (box {64, 64})
  CUtensorMap tm_ws_mn;   // W_s [V, H] bf16 as MN-major B (box {64, 64})
  CUtensorMap tm_dw;      // dW_s [V, H] fp32 output (box {32, 32})
  CUtensorMap tm_dh;      // dHc [N, H] fp32 output (box {32, 32})
  int* tile_counter;      // zeroed before the launch; dynamic tile scheduler
  int N, H, cw, cv0;
  const int32_t* n_dev;   // live row count on the device (nullable: N exact)
  float* dw;              // dW_s [V, H] fp32 (the tm_dw tensor)
  float* dh;              // dHc [dh_rows, H] fp32 (the tm_dh tensor)
  int dw_rows, dh_rows;   // V and the rows of dHc
  int MTW, NT, nW, KBH;
  int dh_accumulate;
};

size_t fused_smem_bytes(int ng, bool dz);
size_t grad_smem_bytes();
cudaError_t tc_setup(int device);  // one-time cudaFuncSetAttribute per device
cudaError_t launch_fused(int ng, bool dz, const FusedArgs& a, int grid, cudaStream_t s);  // grid: CTAs, even
// Top-k estimator: write z_s and z_t (fp32) of the rows of a (variant 1), or
// the top-k dz chunk (variant 2).  ng = 2: hidden payload (both logits by the
// tensor core); ng = 1: logits payload (z_t read from the shipped logits).
cudaError_t launch_fused_topk(int variant, int ng, const FusedArgs& a, int grid, cudaStream_t s);
cudaError_t launch_grad(const GradArgs& a, int grid, cudaStream_t s);
cudaError_t read_and_clear_device_error(int* code);
// RKL_DEBUG build: line of the first failed bounds check in each kernel file
// since the last read (0: none), cleared by the read.
cudaError_t read_and_clear_bounds_tc(int* line);
cudaError_t read_and_clear_bounds_small(int* line);

// ---------------------------------------------------------------- small kernels
cudaError_t launch_compact(const uint8_t* mask, long long T, int32_t* row_idx, int32_t* n_dev, cudaStream_t s);
// hc[p] = h[row_idx[k]] with k = slot_k[p] (slot_k nullptr: k = p); k < 0 gives a zero row.
// With n_dev, rows [n, n rounded up to 256) of hc are zeroed (the padding of
// the last pair tile, read by the tensor-core kernels).
// T: rows of h (the debug build checks every row_idx entry against it).
cudaError_t launch_gather(const void* h_s, const void* h_t, void* hc_s, void* hc_t, const int32_t* row_idx,
                          const int32_t* slot_k, int n_rows, const int32_t* n_dev, int row_bytes, long long T,
                          cudaStream_t s);
// rows: rows of the logits (debug-build check of row_idx).
cudaError_t launch_teacher_lse(const void* logits, bool bf16, const int32_t* row_idx, int N, const int32_t* n_dev,
                               int V, long long pitch, float* lse_t, long long rows, cudaStream_t s);
// Statistics rows p < n_rows are written to compact row slot_k[p] (nullptr: p; < 0: skipped).
cudaError_t launch_combine(const float* part, int S, int n_pad, int n_rows, const int32_t* n_dev,
                           bool teacher_from_part, const float* lse_t_ext, const float* tlogit, float* saved,
                           float* ent_rows, float* lp_rows, const int32_t* slot_k, cudaStream_t s);
cudaError_t launch_scatter_loss(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, long long T,
                                float* loss_tok, cudaStream_t s);
// out[t] = rows[k] where t = row_idx[k], else 0 (per-token [B, S-1] scatter)
cudaError_t launch_scatter_rows(const float* rows, const int32_t* row_idx, int N, const int32_t* n_dev, long long T,
                                float* out, cudaStream_t s);
cudaError_t launch_reduce(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, int B, int Sm1,
                          int reduction, float* loss, cudaStream_t s);
cudaError_t launch_row_weights(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, int n_pad,
                               int B, int Sm1, int reduction, const float* grad_loss, const float* grad_tok,
                               float* rowc, const int32_t* slot_k, cudaStream_t s);
// dH_s[row_idx[k]] = dHc[k_slot[k]] (k_slot nullptr: k), all other rows 0.
cudaError_t launch_scatter_dh(const float* dHc, const int32_t* row_idx, const int32_t* k_slot, int N,
                              const int32_t* n_dev, long long T, int H, float* dH_s, cudaStream_t s);
// Trainable rows per teacher: counts[g] for g < n_teachers, counts[n_teachers] =
// trainable rows whose index is outside [0, n_teachers).  counts must be zeroed.
cudaError_t launch_count_teachers(const uint8_t* mask, const int32_t* teacher_idx, long long T, int n_teachers,
                                  int32_t* counts, cudaStream_t s);
struct TeacherSlots {
  int n;                      // teachers
  int count[kMaxTeachers];    // trainable rows of each teacher
  int base[kMaxTeachers];     // first slot of each teacher (multiples of 256)
};
// Slot of every compact row k (teacher-grouped, ascending within a teacher):
// slot_k[p] = k (slot_k pre-filled with -1 for padding), k_slot[k] = p.
cudaError_t launch_build_slots(const int32_t* row_idx, const int32_t* teacher_idx, int N, const TeacherSlots& ts,
                               int32_t* slot_k, int32_t* k_slot, cudaStream_t s);
cudaError_t launch_pair_fwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx, int N,
                            const int32_t* n_dev, int V, float* saved, cudaStream_t s);
cudaError_t launch_pair_bwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx, int N,
                            const int32_t* n_dev, int n_pad, long long T, int V, const float* rowc, void* dz,
                            cudaStream_t s);

// Top-k estimator with both sides as logits (topk_kernels.cu).  saved [N, 3]
// (lse_s, lse_t, estimate), saved_tk [N, 4] (C, a, K* bits, v_last bits).
// Logit rows: zs + row * zpitch with row = row_idx[k] (local = false) or the
// block-local k (local = true); the sampled token is targets[row_idx[k]].
// The rows of this launch are compacted rows n_base .. n_base + N - 1 (with
// n_dev: as many of them as are live).
cudaError_t launch_topk_fwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, const int32_t* n_dev, int n_base, int V, long long k,
                            float* saved, float* saved_tk, long long zpitch, bool local, cudaStream_t s);
// Top-k forward on the teacher-logits payload: the block's fp32 student
// logits (block-local rows, pitch zpitch) beside the shipped bf16 teacher
// logits (token rows row_idx[kr], pitch tpitch).
cudaError_t launch_topk_fwd_tlogits(const float* zs, const uint16_t* teacher, long long tpitch,
                                    const int32_t* row_idx, const int32_t* targets, int N, const int32_t* n_dev,
                                    int n_base, int V, long long k, float* saved, float* saved_tk, long long zpitch,
                                    cudaStream_t s);
cudaError_t launch_topk_rowk(const float* saved, const float* saved_tk, const int32_t* row_idx,
                             const int32_t* targets, int N, const int32_t* n_dev, int n_pad, float* rowk,
                             cudaStream_t s);
cudaError_t launch_topk_bwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, const int32_t* n_dev, int n_pad, long long T, int V,
                            const float* saved, const float* saved_tk, const float* rowc, void* dz, cudaStream_t s);

// ---------------------------------------------------------------- fp32 CUDA-core path
struct SimtArgs {
  const float* as; const float* at;   // compact rows [N, H] (at: hidden payload)
  const float* bs; const float* bt;   // W [V, H] (bt: hidden payload)
  const float* teacher;               // logits payload: [T, V] fp32
  const int32_t* teacher_rows;
  long long teacher_pitch;
  float* part; const float* rowc;
  const int32_t* row_idx; const int32_t* targets; float* tlogit;
  float* dz;                          // dz chunk [N, cw] fp32
  int N, n_pad, H, V, S, IT, vt_base, chunk_v0, cw;
  const int32_t* n_dev;               // live row count on the device (nullable: N exact)
  int ng;
  int tgroups;                        // > 1: bt is the stacked teacher heads [tgroups, V, H]
  int group_row_end[kMaxTeachers];    // rows of teacher g end here (multiples of 32)
};
constexpr int kSimtBN = 32;
cudaError_t launch_simt_fused(bool dz, const SimtArgs& a, dim3 grid, cudaStream_t s);
// C[M, Nc] (+)= sum_k A(m, k) B(k, n); A(m,k) = A[m*sam + k*sak], B(k,n) = B[k*sbk + n*sbn].
// With n_dev, the row count bounds M (live_dim = 1) or K (live_dim = 2).
cudaError_t launch_simt_gemm(const float* A, long long sam, long long sak, const float* B, long long sbk,
                             long long sbn, float* C, long long ldc, int M, int Nc, int K, int accumulate,
                             const int32_t* n_dev, int live_dim, cudaStream_t s);

}  // namespace rkl
