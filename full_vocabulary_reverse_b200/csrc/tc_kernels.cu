// tc_kernels.cu -- tcgen05 (5th-generation tensor core) kernels of the loss.
//
// fused_kernel<NG, DZ>   S3 / S6: per 256-row tile of the compacted rows (one
//   CTA pair), stream 256-wide vocab tiles of the LM head(s) through TMA ->
//   shared memory -> tcgen05.mma -> TMEM, and reduce each tile in the epilogue
//   without ever writing logits to global memory.
//     NG = 2: hidden-state payload, z_s = h_s W_s^T and z_t = h_t W_t^T in two
//             TMEM accumulators ("feat(mopd): add full-vocabulary on-policy
//             distillation", NeMo RL PR #3978, payload bullet 1).
//     NG = 1: logits payload, z_s from the tensor core, z_t read from the
//             shipped teacher logits (payload bullet 2).
//     DZ = false: online per-row statistics m_s, sum e^(z_s-m_s),
//             A = sum e^(z_s-m_s)(z_s-z_t), m_t, sum e^(z_t-m_t) for one vocab
//             split -> L = A/S_s - lse_s + lse_t after the splits are merged.
//     DZ = true: the shared backward of the same page's first implementation
//             note, dL/dz_s = g p_s ((z_s - z_t) + lse_t - lse_s - L), written
//             as a bf16 [N, cw] chunk for the gradient GEMMs.
//
// grad_kernel  S7: grouped persistent GEMM over one vocab chunk,
//     dW_s[chunk] = dz^T hc_s  and  dHc += dz W_s[chunk]
//   (chain rule through z_s = h_s W_s^T), 256 x 512 tiles per CTA pair, fp32
//   accumulators in TMEM, TMA store / TMA reduce-add epilogue.
//
// All kernels run on 2-CTA clusters with tcgen05.mma.cta_group::2 issued by
// one thread of the leader CTA.  Warp roles: warp 0 = TMA producer, warp 1 =
// MMA issuer, warps 2.. = epilogue, 8 warps (320 threads) in the store
// kernels and the logits-payload forward, 16 (576 threads) in the
// hidden-payload forward.  Epilogue warp w reads TMEM lanes 32*(w%4) .. +31,
// i.e. one tile row per thread, and 1 / (E / 4) of the columns for E
// epilogue warps.  Warp 2 also allocates / frees TMEM.
#include <cuda_bf16.h>

#include "bounds.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rkl {

__device__ int g_dev_err = 0;

RKL_DEFINE_BOUNDS_READER(read_and_clear_bounds_tc)

namespace {

constexpr int kThreads = 64 + 32 * 8;  // gradient kernel: producer, MMA, 8 epilogue warps
constexpr int kFusedEpi = 8;        // dz / writer kernels: 2 epilogue warps per TMEM lane quarter

// Epilogue warps of fused_kernel<NG, DZ>: the forward statistics kernel has
// fwd_epi(NG), the kernels with a store epilogue kFusedEpi (their staging
// boxes live in shared memory beside the pipeline stages).
template <int NG, bool DZ>
__host__ __device__ constexpr int fused_epi() { return DZ ? kFusedEpi : fwd_epi(NG); }
template <int NG, bool DZ>
__host__ __device__ constexpr int fused_threads() { return 64 + 32 * fused_epi<NG, DZ>(); }
constexpr int kStgBoxBytes = 4096;  // one 32-row staging box per epilogue warp

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int bit) {
  atomicOr(&g_dev_err, bit);
  *abort_flag = 1;
}

// Per-CTA shared-memory layout of one pipeline stage of the pair kernel: this
// CTA's 128 rows of A (the compacted hidden rows of z_s and, for NG = 2, of
// z_t) and its half (128 rows) of the 256-row LM-head tile(s), as 64-deep
// boxes [A | B | A' | B'].  NG = 2: (A', B') are z_t's operands at the same K
// (K_STEP = 64).  NG = 1: (A', B') are z_s's operands 64 deeper (K_STEP = 128),
// so that every stage carries eight 256 x 256 x 16 MMAs in both forms: with
// four MMAs per stage the issue loop measured 665 instead of 512 SM cycles
// per 64-deep step, with eight it keeps the tensor pipe busy.  TMEM holds z_s
// (and z_t) for 256 vocab columns: one accumulator slot of 512 columns for
// NG = 2, two slots of 256 for NG = 1.
template <int NG>
struct FusedCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;          // 16 KB
  static constexpr int B_BYTES = (kFBN / 2) * kBK * 2;   // 16 KB
  static constexpr int STAGE_BYTES = 2 * (A_BYTES + B_BYTES);
  static constexpr int K_STEP = NG == 2 ? kBK : 2 * kBK;
  static constexpr int STAGES = 3;
  static constexpr int ACC_COLS = NG * kFBN;
  static constexpr int NUM_ACC = NG == 2 ? 1 : 2;
  static constexpr int TMEM_COLS = NUM_ACC * ACC_COLS;   // 512
};

// Bytes: 1024 alignment slack + stages + epilogue staging + barriers.
template <int NG, bool DZ>
constexpr size_t fused_smem() {
  return 1024 + size_t(FusedCfg<NG>::STAGES) * FusedCfg<NG>::STAGE_BYTES + (DZ ? kFusedEpi * kStgBoxBytes : 0) + 256;
}

// ---- online statistics of one 32-column chunk (all columns valid)
struct RowStats {
  float m_s, S_s, A, m_t, S_t, Bz;  // Bz = sum e^(z_s - m_s) z_s (student entropy)
};

__device__ __forceinline__ void stats_chunk(RowStats& st, const float* zs, const float* zt) {
  float cm_s = zs[0], cm_t = zt[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) {
    cm_s = fmaxf(cm_s, zs[j]);
    cm_t = fmaxf(cm_t, zt[j]);
  }
  const float nm_s = fmaxf(st.m_s, cm_s), nm_t = fmaxf(st.m_t, cm_t);
  const float a_s = ex2((st.m_s - nm_s) * kLog2e), a_t = ex2((st.m_t - nm_t) * kLog2e);
  st.S_s *= a_s;
  st.A *= a_s;
  st.Bz *= a_s;
  st.S_t *= a_t;
  st.m_s = nm_s;
  st.m_t = nm_t;
  const float ms2 = nm_s * kLog2e, mt2 = nm_t * kLog2e;
  float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f, q0 = 0.f, q1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float e0 = ex2(fmaf(zs[j], kLog2e, -ms2));
    const float f0 = ex2(fmaf(zt[j], kLog2e, -mt2));
    const float e1 = ex2(fmaf(zs[j + 1], kLog2e, -ms2));
    const float f1 = ex2(fmaf(zt[j + 1], kLog2e, -mt2));
    s0 += e0;
    t0 += f0;
    q0 = fmaf(e0, zs[j] - zt[j], q0);
    b0 = fmaf(e0, zs[j], b0);
    s1 += e1;
    t1 += f1;
    q1 = fmaf(e1, zs[j + 1] - zt[j + 1], q1);
    b1 = fmaf(e1, zs[j + 1], b1);
  }
  st.S_s += s0 + s1;
  st.S_t += t0 + t1;
  st.A += q0 + q1;
  st.Bz += b0 + b1;
}

// Same for a chunk whose first nv (< 32) columns are inside the vocabulary
// (fully unrolled with predicates so that zs / zt stay in registers).
__device__ __forceinline__ void stats_chunk_tail(RowStats& st, const float* zs, const float* zt, int nv) {
  float cm_s = -INFINITY, cm_t = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (j < nv) {
      cm_s = fmaxf(cm_s, zs[j]);
      cm_t = fmaxf(cm_t, zt[j]);
    }
  const float nm_s = fmaxf(st.m_s, cm_s), nm_t = fmaxf(st.m_t, cm_t);
  const float a_s = ex2((st.m_s - nm_s) * kLog2e), a_t = ex2((st.m_t - nm_t) * kLog2e);
  st.S_s *= a_s;
  st.A *= a_s;
  st.Bz *= a_s;
  st.S_t *= a_t;
  st.m_s = nm_s;
  st.m_t = nm_t;
  const float ms2 = nm_s * kLog2e, mt2 = nm_t * kLog2e;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (j < nv) {
      const float e = ex2(fmaf(zs[j], kLog2e, -ms2));
      const float f = ex2(fmaf(zt[j], kLog2e, -mt2));
      st.S_s += e;
      st.S_t += f;
      st.A = fmaf(e, zs[j] - zt[j], st.A);
      st.Bz = fmaf(e, zs[j], st.Bz);
    }
}

// z_s of the target column if it falls in this 32-column chunk (rare: one
// chunk per row), written once per row.
__device__ __forceinline__ void pick_target(const float* zs, int tgt, int col0, float* out) {
  const unsigned d = static_cast<unsigned>(tgt - col0);
  if (d < 32u) {
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) v = (d == static_cast<unsigned>(j)) ? zs[j] : v;
    *out = v;
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

}  // namespace

// ============================================================================
// Fused forward-statistics / dz kernel on CTA pairs.
//
// A 2-CTA cluster computes a 256-row x 256-column tile of z_s (and z_t) with
// tcgen05.mma.cta_group::2 (M = 256, N = 256): CTA rank r stages rows
// [128 r, 128 r + 128) of the compacted hidden rows and rows
// [128 r, 128 r + 128) of the 256-row LM-head tile, and receives its 128 rows
// of the logits in its own TMEM.  Each staged hidden-row tile feeds 256
// vocab columns, which keeps the operand bytes per flop -- the limit of
// these kernels -- at 1/3 below a 128-column tile.  The
// leader (rank 0) issues the MMAs and owns the operand-full and
// accumulator-empty barriers; both CTAs run the same producer and epilogue
// code on their own rows.
// ============================================================================
// VAR (with DZ = true) selects the epilogue of the top-k estimator: 1 writes
// the z_s and z_t tiles (fp32; with NG = 1, z_t is the exact fp32 value of the
// shipped bf16 teacher logit), 2 writes the top-k dz
// g (p_s ([v in S](w + 1) - C) + [v = y] a),  S = {key(z_s) > K*, or
// key(z_s) = K* and v <= v_last} with the order-preserving float key.
template <int NG, bool DZ, int VAR = 0>
__global__ void __launch_bounds__(fused_threads<NG, DZ>(), 1) fused_kernel(const __grid_constant__ FusedArgs p) {
  using Cfg = FusedCfg<NG>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stg = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + (DZ ? kFusedEpi * kStgBoxBytes : 0));
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* tear = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tear + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  static_assert(Cfg::TMEM_COLS <= 512, "TMEM has 512 columns");
  // Rows of this launch: exact, or read from the device (both CTAs of a pair
  // read the same value, so they walk the same units).
  const int n_rows = live_rows(p.n_dev, p.N, p.n_base);
  const int MT = (n_rows + 2 * kBM - 1) / (2 * kBM);
  const int units_total = MT * p.G;
  const int n_ksteps = (p.KB * kBK + Cfg::K_STEP - 1) / Cfg::K_STEP;  // pipeline stages per vocab tile

  // Work of this pair: units u = pair, pair + npairs, ...
  // Unit u = (256-row tile u % MT, vocab group u / MT); group g covers the
  // vocab tiles vt_base + [g*GT, min(g*GT + GT, IT)).  With the row tile as
  // the fast index, the pairs running at any moment share a few vocab groups,
  // so each LM-head tile is fetched from HBM once and re-served from L2 to
  // every row tile.  Forward statistics are flushed per unit, so their
  // grouping depends on V only -- never on N or on the grid -- and a row's
  // loss does not depend on the rest of the batch.

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * fused_epi<NG, DZ>());  // every epilogue warp of both CTAs
    }
    mbar_init(tear, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_as);
      tma_prefetch_desc(&p.tm_bs);
      if (NG == 2) {
        tma_prefetch_desc(&p.tm_at);
        tma_prefetch_desc(&p.tm_bt);
      }
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);  // leader's full[0]
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;  // bit i: stage i has been armed at least once
      uint32_t last_par = 0;
      bool ok = true;
      for (int u = pair; u < units_total && ok; u += npairs) {
        const int m0 = (u % MT) * 2 * kBM + rank * kBM;
        const int g = u / MT;
        const int vt_end = min(g * p.GT + p.GT, p.IT);
        // Teacher per row: the head of this tile's teacher starts at row
        // teacher * V of the stacked heads.  Columns at or past V of a tile
        // then read the next head's rows instead of zeros; the epilogue never
        // uses them (statistics stop at V, the dz store is clipped at V).
        int tv_off = 0;
        if (NG == 2 && p.tgroups > 1) {
          const int tile_row = (u % MT) * 2 * kBM;
          int tg = 0;
          while (tg + 1 < p.tgroups && tile_row >= p.group_row_end[tg]) ++tg;
          tv_off = tg * p.V;
        }
        for (int vt = g * p.GT; vt < vt_end && ok; ++vt) {
          const int v0 = (p.vt_base + vt) * kFBN + rank * (kFBN / 2);
          for (int kb = 0; kb < n_ksteps; ++kb) {
            const int k0 = kb * Cfg::K_STEP;
            if (!mbar_wait_cluster(&empty[stage], phase ^ 1, abort_flag)) {
              raise_abort(abort_flag, ERR_WAIT_TMA_EMPTY);
              ok = false;
              break;
            }
            // TMA coordinates: x (the K offset) on a 16-byte boundary inside H,
            // rows inside the padded row layout, vocab rows inside the launch
            if (!RKL_BOUNDS((k0 & 7) == 0 && k0 < p.H && m0 >= 0 && m0 < p.n_pad && v0 >= 0 &&
                            v0 < (p.vt_base + p.IT) * kFBN && tv_off >= 0 &&
                            tv_off <= (p.tgroups > 1 ? (p.tgroups - 1) * p.V : 0))) {
              raise_abort(abort_flag, ERR_BOUNDS);
              ok = false;
              break;
            }
            uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
            const uint32_t fb = full0 + stage * 8;
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
            tma_load_2d_pair(sa, &p.tm_as, fb, k0, m0);
            tma_load_2d_pair(sa + Cfg::A_BYTES, &p.tm_bs, fb, k0, v0);
            if (NG == 2) {
              tma_load_2d_pair(sa + Cfg::A_BYTES + Cfg::B_BYTES, &p.tm_at, fb, k0, m0);
              tma_load_2d_pair(sa + 2 * Cfg::A_BYTES + Cfg::B_BYTES, &p.tm_bt, fb, k0, v0 + tv_off);
            } else {
              // the next 64 of K; past H (odd H / 64) the boxes are zero-filled
              // (x = H is on a 16-byte boundary) and their MMAs add zeros
              tma_load_2d_pair(sa + Cfg::A_BYTES + Cfg::B_BYTES, &p.tm_as, fb, k0 + kBK, m0);
              tma_load_2d_pair(sa + 2 * Cfg::A_BYTES + Cfg::B_BYTES, &p.tm_bs, fb, k0 + kBK, v0);
            }
            armed |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
      // The leader's full barriers count both CTAs' loads: drain them there.
      if (leader)
        for (int i = 0; i < STAGES; ++i)
          if (armed & (1u << i)) {
            volatile int never = 0;
            if (!mbar_wait(&full[i], (last_par >> i) & 1, &never)) atomicOr(&g_dev_err, ERR_WAIT_TEARDOWN);
          }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * kBM, kFBN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int u = pair; u < units_total && ok; u += npairs) {
        const int g = u / MT;
        const int vt_end = min(g * p.GT + p.GT, p.IT);
        for (int vt = g * p.GT; vt < vt_end && ok; ++vt, ++it) {
          const int acc = it % Cfg::NUM_ACC;
          const uint32_t ap = (it / Cfg::NUM_ACC) & 1;
          if (!mbar_wait_cluster(&acc_empty[acc], ap ^ 1, abort_flag)) {
            raise_abort(abort_flag, ERR_WAIT_ACC_EMPTY);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_s = tmem_base + acc * Cfg::ACC_COLS;
          const uint32_t d_t = d_s + kFBN;
          for (int kb = 0; kb < n_ksteps; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) {
              raise_abort(abort_flag, ERR_WAIT_TMA_FULL);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES);
            const uint32_t sb = sa + Cfg::A_BYTES;
            const uint32_t sat = sb + Cfg::B_BYTES;
            const uint32_t sbt = sat + Cfg::A_BYTES;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint32_t acc_flag = (kb | k) != 0;
              umma_bf16_pair(d_s, sdesc_sw128(sa + 32 * k, 16, 1024), sdesc_sw128(sb + 32 * k, 16, 1024), idesc,
                             acc_flag);
              if (NG == 2)
                umma_bf16_pair(d_t, sdesc_sw128(sat + 32 * k, 16, 1024), sdesc_sw128(sbt + 32 * k, 16, 1024),
                               idesc, acc_flag);
            }
            if (NG == 1) {
              // K order kept: the second box follows the first
#pragma unroll
              for (int k = 0; k < kBK / 16; ++k)
                umma_bf16_pair(d_s, sdesc_sw128(sat + 32 * k, 16, 1024), sdesc_sw128(sbt + 32 * k, 16, 1024), idesc,
                               1u);
            }
            umma_commit_pair(&empty[stage], 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (ok) umma_commit_pair(&acc_full[acc], 0x3);
        }
      }
      // All issued MMAs must finish before TMEM is released.
      umma_commit_pair(tear, 0x1);
      volatile int never = 0;
      if (!mbar_wait(tear, 0, &never)) atomicOr(&g_dev_err, ERR_WAIT_TEARDOWN);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quarter q = w % 4 (tile rows 32 q .. 32 q + 31)
    // and columns [128 h, 128 h + 128) of the 256-column tile, h = (w-2) / 4.
    const int q = warp & 3;
    // Warp part p = (w - 2) / 4 owns columns [COLS p, COLS p + COLS).
    constexpr int COLS = kFBN / (fused_epi<NG, DZ>() / 4);
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    int cur_m0 = -1;
    float lse2 = 0.f, cst = 0.f, g_row = 0.f;
    float tk_C = 0.f, tk_ga = 0.f;     // top-k dz: C and g a
    float tk_thr = 0.f;  // top-k dz: the support bound K* as a float
    int tk_vlast = -1, tk_y = -1;
    int tgt = -1;  // target column of this row (forward with targets), else -1
    const uint16_t* trow = nullptr;
    int box = 0;
    int it = 0;
    bool ok = true;
    for (int u = pair; u < units_total && ok; u += npairs) {
      const int m0 = (u % MT) * 2 * kBM + rank * kBM;  // this CTA's first row
      const int g = u / MT;
      const int vt_end = min(g * p.GT + p.GT, p.IT);
      if (m0 != cur_m0) {
        cur_m0 = m0;
        const int r = m0 + row;
        if (DZ && VAR == 2) {
          lse2 = p.rowc[r];
          g_row = p.rowc[2 * p.n_pad + r];
          cst = p.rowk[r];
          tk_C = p.rowk[p.n_pad + r];
          tk_ga = g_row * p.rowk[2 * p.n_pad + r];
          // K* is an order-preserving key (-0 and +0 one key); as a float the
          // test key(z) > K* is z > thr and key(z) = K* is z == thr (IEEE
          // compares -0 == +0).  K* = 0 (below every key: the whole row) is
          // -inf; K* = ~0 (above every key: no member) decodes to a NaN, which
          // no compare passes.
          const uint32_t kk = __float_as_uint(p.rowk[3 * p.n_pad + r]);
          tk_thr = kk == 0u ? -INFINITY : __uint_as_float((kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk);
          tk_vlast = __float_as_int(p.rowk[4 * p.n_pad + r]);
          tk_y = __float_as_int(p.rowk[5 * p.n_pad + r]);
        } else if (DZ && VAR == 0) {
          lse2 = p.rowc[r];
          cst = p.rowc[p.n_pad + r];
          g_row = p.rowc[2 * p.n_pad + r];
        } else if (!DZ) {
          tgt = (p.targets != nullptr && r < n_rows) ? p.targets[p.row_idx[r]] : -1;
        }
        if (NG == 1) {
          // the top-k writer of the logits payload stores z_s only (the
          // selection reads the shipped teacher rows itself): no teacher row
          trow = nullptr;
          if (r < n_rows && !(DZ && VAR == 1)) {
            const long long tr = p.teacher_rows ? p.teacher_rows[r] : r;
            trow = p.teacher + tr * p.teacher_pitch;
          }
        }
      }
      RowStats st{-INFINITY, 0.f, 0.f, -INFINITY, 0.f, 0.f};
      for (int vt = g * p.GT; vt < vt_end; ++vt, ++it) {
        const int v0 = (p.vt_base + vt) * kFBN + half * COLS;  // this warp's first column
        // Teacher logits of this row (logits payload): 32 bf16 per chunk,
        // loaded one chunk ahead.
        uint4 tcur[NG == 1 ? 4 : 1], tnxt[NG == 1 ? 4 : 1];
        if (NG == 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tcur[i] = (trow != nullptr && i * 8 < p.V - v0) ? ldg_nc_v4(trow + v0 + i * 8) : make_uint4(0, 0, 0, 0);
          }
        }
        const int acc = it % Cfg::NUM_ACC;
        const uint32_t ap = (it / Cfg::NUM_ACC) & 1;
        bool w_ok = mbar_wait_cluster(&acc_full[acc], ap, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) {
          if (lane == 0) raise_abort(abort_flag, ERR_WAIT_ACC_FULL);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem_base + lane_off + acc * Cfg::ACC_COLS + half * COLS;
        constexpr int kChunks = COLS / 32;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          float zs[32], zt[32];
          if (NG == 1 && c + 1 < kChunks) {
            const int vn = v0 + (c + 1) * 32;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              tnxt[i] = (trow != nullptr && i * 8 < p.V - vn) ? ldg_nc_v4(trow + vn + i * 8) : make_uint4(0, 0, 0, 0);
          }
          tmem_ld_32x32(tb + c * 32, zs);
          if (NG == 2) tmem_ld_32x32(tb + kFBN + c * 32, zt);
          tmem_wait_ld();
          if (c == kChunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0 + acc * 8);
          }
          if (NG == 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 w = tcur[i];
              zt[8 * i + 0] = bf16_lo(w.x);
              zt[8 * i + 1] = bf16_hi(w.x);
              zt[8 * i + 2] = bf16_lo(w.y);
              zt[8 * i + 3] = bf16_hi(w.y);
              zt[8 * i + 4] = bf16_lo(w.z);
              zt[8 * i + 5] = bf16_hi(w.z);
              zt[8 * i + 6] = bf16_lo(w.w);
              zt[8 * i + 7] = bf16_hi(w.w);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) tcur[i] = tnxt[i];
          }
          if (!DZ) {
            const int nv = p.V - (v0 + c * 32);
            if (nv >= 32)
              stats_chunk(st, zs, zt);
            else if (nv > 0)
              stats_chunk_tail(st, zs, zt, nv);
            if (tgt >= 0 && RKL_BOUNDS(m0 + row < p.n_pad)) pick_target(zs, tgt, v0 + c * 32, p.tlogit + m0 + row);
          } else if (VAR == 1) {
            // z_s (and, NG = 2, z_t) of this 32-column chunk, fp32, one 32 x 32
            // box each (columns past V are clipped by the TMA store)
            uint8_t* buf = stg + (warp - 2) * kStgBoxBytes;  // one staging box per warp
#pragma unroll
            for (int which = 0; which < NG; ++which) {
              const float* src = which == 0 ? zs : zt;
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
              const uint32_t rbase = smem_u32(buf) + lane * 128;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                st_shared_v4(rbase + ((e ^ (lane & 7)) << 4), __float_as_uint(src[4 * e]),
                             __float_as_uint(src[4 * e + 1]), __float_as_uint(src[4 * e + 2]),
                             __float_as_uint(src[4 * e + 3]));
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0 && RKL_BOUNDS(v0 + c * 32 >= 0 && m0 + q * 32 >= 0)) {
                tma_store_2d(which == 0 ? &p.tm_zs : &p.tm_zt, buf, v0 + c * 32, m0 + q * 32);
                bulk_commit();
              }
            }
          } else {
            // dz = g * p_s * ((z_s - z_t) + cst); columns past the chunk end
            // are clipped by the TMA store.
            uint32_t pk[16];
            if (VAR == 2) {
              // top-k: dz = g p_s ([v in S](w + 1) - C) + [v = y] g a
              const int col0 = v0 + c * 32;
              const int vl = tk_vlast - col0, yo = tk_y - col0;  // offsets in this chunk
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                float d[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const float x = zs[j + h];
                  const bool in = x > tk_thr || (x == tk_thr && j + h <= vl);
                  const float pr = ex2(fmaf(x, kLog2e, -lse2));
                  const float coef = (in ? (x - zt[j + h]) + cst + 1.f : 0.f) - tk_C;
                  d[h] = g_row * pr * coef + (j + h == yo ? tk_ga : 0.f);
                }
                pk[j / 2] = pack_bf16x2(d[0], d[1]);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                const float p0 = ex2(fmaf(zs[j], kLog2e, -lse2));
                const float p1 = ex2(fmaf(zs[j + 1], kLog2e, -lse2));
                const float d0 = g_row * p0 * ((zs[j] - zt[j]) + cst);
                const float d1 = g_row * p1 * ((zs[j + 1] - zt[j + 1]) + cst);
                pk[j / 2] = pack_bf16x2(d0, d1);
              }
            }
            uint8_t* buf = stg + (warp - 2) * kStgBoxBytes;  // one staging box per warp
            if ((c & 1) == 0) {
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
            }
            const uint32_t rbase = smem_u32(buf) + lane * 128;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int chunk16 = (c & 1) * 4 + i;
              st_shared_v4(rbase + ((chunk16 ^ (lane & 7)) << 4), pk[4 * i], pk[4 * i + 1], pk[4 * i + 2],
                           pk[4 * i + 3]);
            }
            if (c & 1) {
              fence_proxy_async_smem();
              __syncwarp();
              // a TMA store must not start at a negative coordinate; x (bf16) on a 16-byte boundary
              const int dx = v0 - p.chunk_v0 + (c - 1) * 32;
              if (lane == 0 && RKL_BOUNDS(dx >= 0 && (dx & 7) == 0 && m0 + q * 32 >= 0)) {
                tma_store_2d(&p.tm_dz, buf, dx, m0 + q * 32);
                bulk_commit();
              }
              ++box;
            }
          }
        }
      }
      if (!DZ && ok && RKL_BOUNDS(m0 + row < p.n_pad && g < p.G)) {
        // statistics slot (group, column part): fwd_slots(NG) slots per group
        float* base = p.part + static_cast<size_t>(fwd_slots(NG) * g + half) * kStatVals * p.n_pad + m0 + row;
        base[0] = st.m_s;
        base[p.n_pad] = st.S_s;
        base[2 * p.n_pad] = st.A;
        base[3 * p.n_pad] = st.m_t;
        base[4 * p.n_pad] = st.S_t;
        base[5 * p.n_pad] = st.Bz;
      }
    }
    if (DZ) {
      if (lane == 0) bulk_wait<0>();
      __syncwarp();
    }
  }

  // Neither CTA may release its TMEM or shared memory while the pair MMAs or
  // the other CTA can still touch them.
  tc_fence_before();
  cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

// ============================================================================
// Grouped gradient GEMM: dW_s tiles (A = dz^T, MN-major; B = hc_s, MN-major)
// then dH tiles (A = dz, K-major; B = W_s, MN-major).  256 x 512 pair tiles.
// ============================================================================
namespace {
constexpr int kGA = kBM * kBK * 2;           // 16 KB: this CTA's 128 rows of A
constexpr int kGBP = 128 * kBK * 2;          // 16 KB: one 128-column piece of B
constexpr int kGStage = kGA + 2 * kGBP;      // 48 KB: A + this CTA's two B pieces
constexpr int kGStages = 4;
constexpr int kGTmemCols = kGradBN;          // 512: one 256 x 512 accumulator (two N = 256 halves)
constexpr int kSched = 2;                    // tile-index broadcast ring depth
}  // namespace

// One 2-CTA cluster computes a 256 x 512 tile as two tcgen05.mma.cta_group::2
// products of N = 256 that share the A operand: CTA rank r holds rows
// [128 r, 128 r + 128) of A, and for half j = 0, 1 the columns
// [256 j + 128 r, 256 j + 128 r + 128) of B, and receives rows
// [128 r, 128 r + 128) of D in its own TMEM (columns [256 j, 256 j + 256) =
// half j).  Per 64-deep K step a CTA streams 48 KB (16 KB of A, 32 KB of B)
// for 2 x 256 x 256 x 64 x 2 flop, a third fewer bytes per flop than a
// 256 x 256 tile; that matters because these kernels are bound by the
// L2 -> shared-memory operand feed.  TMEM holds the whole 512-column tile, so
// the epilogue drains it in two halves: half 0 (all eight epilogue warps)
// first, then half 1, and the next tile's first MMA into a half waits only
// for that half.  The leader (rank 0) issues the MMAs and owns the
// operand-full barriers (both CTAs' TMA loads count on them), the
// accumulator barriers (both CTAs' epilogues arrive) and the tile scheduler
// (it claims tiles with an atomic counter and writes each index into both
// CTAs' rings).
__global__ void __launch_bounds__(kThreads, 1) grad_kernel(const __grid_constant__ GradArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stg = smem + kGStages * kGStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + 8 * kStgBoxBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGStages;
  uint64_t* acc_full = bars + 2 * kGStages;
  uint64_t* acc_empty = acc_full + 1;  // [2]: one per accumulator half
  uint64_t* tear = acc_empty + 2;
  uint64_t* sched_full = tear + 1;             // [kSched]
  uint64_t* sched_empty = sched_full + kSched;  // [kSched]
  int* sched_tile = reinterpret_cast<int*>(sched_empty + kSched);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched_tile + kSched);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // Row count (exact, or read from the device): dH tiles cover the rows in
  // 256-row pair tiles, dW tiles reduce over them in 64-row K steps.  With no
  // live row the dW tiles have K = 0 and store zeros.
  const int n_rows = live_rows(p.n_dev, p.N);
  const int nH = ((n_rows + 2 * kBM - 1) / (2 * kBM)) * p.NT;
  const int KBW = (n_rows + kBK - 1) / kBK;
  const int n_tiles = p.nW + nH;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&acc_empty[i], 16);  // 8 epilogue warps in each CTA of the pair
    for (int i = 0; i < kSched; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1 + 8 + 1 + 8);  // leader MMA + epilogues, peer producer + epilogues
    }
    mbar_init(tear, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_holder, kGTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_dz_k);
      tma_prefetch_desc(&p.tm_dz_mn);
      tma_prefetch_desc(&p.tm_hs_mn);
      tma_prefetch_desc(&p.tm_ws_mn);
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);  // leader's full[0]
      int stage = 0;
      uint32_t phase = 0, armed = 0, last_par = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % kSched;
        const uint32_t sp = (i / kSched) & 1;
        int t;
        if (leader) {
          if (!mbar_wait_cluster(&sched_empty[slot], sp ^ 1, abort_flag)) {
            raise_abort(abort_flag, ERR_WAIT_AUX);
            break;
          }
          t = atomicAdd(p.tile_counter, 1);
          if (t >= n_tiles) t = -1;
          sched_tile[slot] = t;
          st_cluster_u32(mapa_shared(smem_u32(&sched_tile[slot]), 1), static_cast<uint32_t>(t));
          mbar_arrive(&sched_full[slot]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&sched_full[slot]), 1));
        } else {
          if (!mbar_wait_cluster(&sched_full[slot], sp, abort_flag)) {
            raise_abort(abort_flag, ERR_WAIT_AUX);
            break;
          }
          t = sched_tile[slot];
          mbar_arrive_cluster(mapa_shared(smem_u32(&sched_empty[slot]), 0));
        }
        if (t < 0) break;
        const bool is_h = t < nH;
        const int tt = is_h ? t : t - nH;
        // tile tt = (row / vocab block tt / NT, H block tt % NT): the H block is
        // the fast index, so the tiles running together share their A block
        // (a slice of dz) in L2 and each slice of dz is read from memory once.
        const int m0 = (tt / p.NT) * 2 * kBM + rank * kBM;   // this CTA's A rows
        const int nb = (tt % p.NT) * kGradBN + rank * 128;   // this CTA's first B piece
        const int KB = is_h ? p.KBH : KBW;
        // tile index and TMA coordinates: x of every load on a 16-byte boundary
        // (m0 is the x of the dz^T loads), no negative row of W_s
        if (!RKL_BOUNDS(t < n_tiles && tt >= 0 && m0 >= 0 && (m0 & 7) == 0 && (nb & 7) == 0 &&
                        nb < p.NT * kGradBN && p.cv0 >= 0)) {
          raise_abort(abort_flag, ERR_BOUNDS);
          break;
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1, abort_flag)) {
            raise_abort(abort_flag, ERR_WAIT_TMA_EMPTY);
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * kGStage;
          uint8_t* sb = sa + kGA;
          const uint32_t fb = full0 + stage * 8;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kGStage);
          if (!is_h) {
            // A = dz^T: two 64-wide vocab blocks x 64 rows (K); B = hc_s.
            tma_load_2d_pair(sa, &p.tm_dz_mn, fb, m0, kb * kBK);
            tma_load_2d_pair(sa + kGA / 2, &p.tm_dz_mn, fb, m0 + 64, kb * kBK);
          } else {
            // A = dz (K-major); B = W_s rows of the chunk.
            tma_load_2d_pair(sa, &p.tm_dz_k, fb, kb * kBK, m0);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint8_t* bp = sb + j * kGBP;
            const int n = nb + j * (kGradBN / 2);
            if (!is_h) {
              tma_load_2d_pair(bp, &p.tm_hs_mn, fb, n, kb * kBK);
              tma_load_2d_pair(bp + kGBP / 2, &p.tm_hs_mn, fb, n + 64, kb * kBK);
            } else {
              tma_load_2d_pair(bp, &p.tm_ws_mn, fb, n, p.cv0 + kb * kBK);
              tma_load_2d_pair(bp + kGBP / 2, &p.tm_ws_mn, fb, n + 64, p.cv0 + kb * kBK);
            }
          }
          armed |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kGStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // The leader's full barriers count both CTAs' loads: drain them there.
      if (leader)
        for (int i = 0; i < kGStages; ++i)
          if (armed & (1u << i)) {
            volatile int never = 0;
            if (!mbar_wait(&full[i], (last_par >> i) & 1, &never)) atomicOr(&g_dev_err, ERR_WAIT_TEARDOWN);
          }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      constexpr uint32_t idesc_w = idesc_bf16(2 * kBM, kGradBN / 2, 1, 1);
      constexpr uint32_t idesc_h = idesc_bf16(2 * kBM, kGradBN / 2, 0, 1);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % kSched;
        const uint32_t sp = (i / kSched) & 1;
        if (!mbar_wait(&sched_full[slot], sp, abort_flag)) {
          raise_abort(abort_flag, ERR_WAIT_AUX);
          break;
        }
        const int t = sched_tile[slot];
        mbar_arrive(&sched_empty[slot]);
        if (t < 0) break;
        const bool is_h = t < nH;
        const int KB = is_h ? p.KBH : KBW;
        const uint32_t ap = i & 1;  // the accumulator is drained once per tile
        // The tile kind selects A's layout once per tile: dH tiles read dz
        // K-major (a 16-deep K slice is 32 B along the swizzled row), dW tiles
        // read dz^T MN-major (a slice is 16 rows of 128 B; the two 64-wide
        // vocab blocks lie kGA / 2 apart).  Keeping the choice out of the K
        // loop leaves the MMA issue free of branches: a per-MMA branch on the
        // kind measured 1330 instead of 1113 SM cycles per 64-deep K step.
        const uint32_t idesc = is_h ? idesc_h : idesc_w;
        const uint32_t a_step = is_h ? 32u : 2048u;
        const uint32_t a_lbo = is_h ? 16u : static_cast<uint32_t>(kGA / 2);
        if (KB == 0) {
          // No K step (no live row): no MMA, the epilogue stores zeros; the
          // accumulator hand-off still waits for both halves to be drained.
          for (int j = 0; j < 2 && ok; ++j)
            if (!mbar_wait_cluster(&acc_empty[j], ap ^ 1, abort_flag)) {
              raise_abort(abort_flag, ERR_WAIT_ACC_EMPTY);
              ok = false;
            }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            raise_abort(abort_flag, ERR_WAIT_TMA_FULL);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kGStage);
          const uint32_t sb = sa + kGA;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (kb == 0) {
              // the previous tile's epilogue must have read this half out
              if (!mbar_wait_cluster(&acc_empty[j], ap ^ 1, abort_flag)) {
                raise_abort(abort_flag, ERR_WAIT_ACC_EMPTY);
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint32_t d = tmem_base + j * (kGradBN / 2);
            const uint32_t bj = sb + j * kGBP;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16_pair(d, sdesc_sw128(sa + a_step * k, a_lbo, 1024), sdesc_sw128(bj + 2048 * k, kGBP / 2, 1024),
                             idesc, (kb | k) != 0);
          }
          if (!ok) break;
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == kGStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit_pair(acc_full, 0x3);
      }
      umma_commit_pair(tear, 0x1);
      volatile int never = 0;
      if (!mbar_wait(tear, 0, &never)) atomicOr(&g_dev_err, ERR_WAIT_TEARDOWN);
    }
  } else {
    // Warp w reads TMEM lane quarter w % 4.  Half 0 of the accumulator is
    // drained first by all eight warps (warp w takes columns
    // [128 s, 128 s + 128) of the half, s = (w - 2) / 4), then half 1.
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t sched_empty0 = mapa_shared(smem_u32(sched_empty), 0);
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t* buf = stg + (warp - 2) * kStgBoxBytes;  // one staging box per warp
    for (int i = 0;; ++i) {
      const int slot = i % kSched;
      const uint32_t sp = (i / kSched) & 1;
      bool ok = mbar_wait_cluster(&sched_full[slot], sp, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_abort(abort_flag, ERR_WAIT_AUX);
        break;
      }
      const int t = sched_tile[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sched_empty0 + slot * 8);
      if (t < 0) break;
      const bool is_h = t < nH;
      const int tt = is_h ? t : t - nH;
      const int mtile = tt / p.NT;
      const int n0 = (tt % p.NT) * kGradBN;
      ok = mbar_wait_cluster(acc_full, i & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) raise_abort(abort_flag, ERR_WAIT_ACC_FULL);
        break;
      }
      tc_fence_after();
      const int rows = mtile * 2 * kBM + rank * kBM + q * 32;
      const int row0 = is_h ? rows : p.cv0 + rows;
      const bool zero_acc = !is_h && KBW == 0;  // no K step: the tile is zero
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        const int col = j * (kGradBN / 2) + sub * 128;  // first column of this warp in the tile
        const uint32_t tb = tmem_base + lane_off + col;
        // all 128 columns of this warp's part of the half in one burst, so the
        // half is released to the next tile's MMAs before any staging work
        float vv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32(tb + c * 32, vv[c]);
        tmem_wait_ld();
        if (zero_acc) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) vv[c][e] = 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + j * 8);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float* v = vv[c];
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          const uint32_t rbase = smem_u32(buf) + lane * 128;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_shared_v4(rbase + ((e ^ (lane & 7)) << 4), __float_as_uint(v[4 * e]), __float_as_uint(v[4 * e + 1]),
                         __float_as_uint(v[4 * e + 2]), __float_as_uint(v[4 * e + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          const int cx = n0 + col + c * 32;
          // fp32 TMA store / reduce: x on a 16-byte boundary, no negative coordinate
          if (lane == 0 && RKL_BOUNDS(cx >= 0 && (cx & 3) == 0 && row0 >= 0)) {
            if (!is_h)
              tma_store_2d(&p.tm_dw, buf, cx, row0);
            else if (p.dh_accumulate)
              tma_reduce_add_2d(&p.tm_dh, buf, cx, row0);
            else
              tma_store_2d(&p.tm_dh, buf, cx, row0);
            bulk_commit();
          }
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  // Neither CTA may release its TMEM or shared memory while the pair MMAs or
  // the other CTA can still touch them.
  tc_fence_before();
  cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kGTmemCols);
  }
}

// ============================================================================
// Host launchers
// ============================================================================
size_t fused_smem_bytes(int ng, bool dz) {
  if (ng == 2) return dz ? fused_smem<2, true>() : fused_smem<2, false>();
  return dz ? fused_smem<1, true>() : fused_smem<1, false>();
}

size_t grad_smem_bytes() { return 1024 + size_t(kGStages) * kGStage + 8 * kStgBoxBytes + 512; }

cudaError_t tc_setup(int /*device*/) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(fused_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<2, false>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<2, true>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<1, false>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<1, true>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<2, true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<2, true>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<2, true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<2, true>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<1, true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<1, true>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(fused_kernel<1, true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fused_smem<1, true>())) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)grad_smem_bytes());
}

template <typename K>
static cudaError_t launch_pair(K kernel, int grid, int threads, size_t smem, cudaStream_t s, const FusedArgs& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid & ~1);  // whole CTA pairs
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_fused(int ng, bool dz, const FusedArgs& a, int grid, cudaStream_t s) {
  const size_t smem = fused_smem_bytes(ng, dz);
  const int id = ng == 2 ? (dz ? K_DZ_DUAL_TC : K_FWD_DUAL_TC) : (dz ? K_DZ_SINGLE_TC : K_FWD_SINGLE_TC);
  LaunchScope scope(id, s);
  if (ng == 2) return dz ? launch_pair(fused_kernel<2, true>, grid, fused_threads<2, true>(), smem, s, a)
                         : launch_pair(fused_kernel<2, false>, grid, fused_threads<2, false>(), smem, s, a);
  return dz ? launch_pair(fused_kernel<1, true>, grid, fused_threads<1, true>(), smem, s, a) : launch_pair(fused_kernel<1, false>, grid, fused_threads<1, false>(), smem, s, a);
}

cudaError_t launch_fused_topk(int variant, int ng, const FusedArgs& a, int grid, cudaStream_t s) {
  const size_t smem = fused_smem_bytes(ng, true);
  if (ng == 2) {
    LaunchScope scope(variant == 1 ? K_ZW_DUAL_TC : K_DZ_TOPK_TC, s);
    return variant == 1 ? launch_pair(fused_kernel<2, true, 1>, grid, fused_threads<2, true>(), smem, s, a)
                        : launch_pair(fused_kernel<2, true, 2>, grid, fused_threads<2, true>(), smem, s, a);
  }
  LaunchScope scope(variant == 1 ? K_ZW_SINGLE_TC : K_DZ_TOPK_SINGLE_TC, s);
  return variant == 1 ? launch_pair(fused_kernel<1, true, 1>, grid, fused_threads<1, true>(), smem, s, a)
                      : launch_pair(fused_kernel<1, true, 2>, grid, fused_threads<1, true>(), smem, s, a);
}

cudaError_t launch_grad(const GradArgs& a, int grid, cudaStream_t s) {
  LaunchScope scope(K_GRAD_TC, s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid & ~1);  // whole CTA pairs
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = grad_smem_bytes();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, grad_kernel, a);
}

cudaError_t read_and_clear_device_error(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_dev_err, sizeof(int));
  if (e != cudaSuccess) return e;
  *code = v;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int));
  }
  return e;
}

}  // namespace rkl
