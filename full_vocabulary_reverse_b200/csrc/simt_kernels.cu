// simt_kernels.cu -- fp32 path of S3 / S6 / S7 on the CUDA cores (FFMA).
//
// The tensor cores have no fp32 input kind, so fp32 problems take this path.
// It is the same algorithm as the tcgen05 kernels -- vocab split statistics
// merged by the same combine kernel, dz rebuilt per vocab chunk, dH/dW as two
// GEMMs -- with 32x32 tiles computed by FFMA into shared memory and one thread
// per row doing the online reduction.  It exists for correctness on fp32
// inputs, not for speed.
#include "kernels.h"
#include "sm100.cuh"

namespace rkl {
namespace {

constexpr int TB = kSimtBN;  // 32

template <bool DZ>
__global__ void __launch_bounds__(256) simt_fused_kernel(const SimtArgs a) {
  __shared__ float As[TB][TB + 1], At[TB][TB + 1], Bs[TB][TB + 1], Bt[TB][TB + 1];
  __shared__ float Zs[TB][TB + 1], Zt[TB][TB + 1];
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;  // ty in 0..7
  const int N = live_rows(a.n_dev, a.N);  // rows in use (exact, or read from the device)

  int u0, u1, split = 0;
  if (!DZ) {
    const int mt = blockIdx.x;
    if (mt * TB >= N) return;
    split = blockIdx.y;
    u0 = mt * a.IT + static_cast<int>((static_cast<long long>(split) * a.IT) / a.S);
    u1 = mt * a.IT + static_cast<int>((static_cast<long long>(split + 1) * a.IT) / a.S);
  } else {
    const int MT = (N + TB - 1) / TB;
    const int total = MT * a.IT;
    u0 = static_cast<int>((static_cast<long long>(blockIdx.x) * total) / gridDim.x);
    u1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * total) / gridDim.x);
  }

  float m_s = -INFINITY, S_s = 0.f, A = 0.f, m_t = -INFINITY, S_t = 0.f, Bz = 0.f;
  int tgt = -1;
  if (!DZ && tid < TB && a.targets != nullptr) {
    const int r = (u0 / a.IT) * TB + tid;
    if (r < N) tgt = a.targets[a.row_idx[r]];
  }
  for (int u = u0; u < u1; ++u) {
    const int m0 = (u / a.IT) * TB;
    const int v0 = (a.vt_base + u % a.IT) * TB;
    // teacher per row: rows of teacher g end at group_row_end[g]
    const float* bt = a.bt;
    if (a.tgroups > 1) {
      int tg = 0;
      while (tg + 1 < a.tgroups && m0 >= a.group_row_end[tg]) ++tg;
      bt += static_cast<long long>(tg) * a.V * a.H;
    }
    float cs[4] = {0.f, 0.f, 0.f, 0.f}, ct[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < a.H; k0 += TB) {
      for (int e = tid; e < TB * TB; e += 256) {
        const int r = e / TB, kk = e % TB;
        const bool kin = k0 + kk < a.H;
        As[r][kk] = (m0 + r < N && kin) ? a.as[static_cast<long long>(m0 + r) * a.H + k0 + kk] : 0.f;
        Bs[r][kk] = (v0 + r < a.V && kin) ? a.bs[static_cast<long long>(v0 + r) * a.H + k0 + kk] : 0.f;
        if (a.ng == 2) {
          At[r][kk] = (m0 + r < N && kin) ? a.at[static_cast<long long>(m0 + r) * a.H + k0 + kk] : 0.f;
          Bt[r][kk] = (v0 + r < a.V && kin) ? bt[static_cast<long long>(v0 + r) * a.H + k0 + kk] : 0.f;
        }
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < TB; ++kk) {
        const float bsv = Bs[tx][kk];
        const float btv = Bt[tx][kk];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          cs[i] = fmaf(As[ty * 4 + i][kk], bsv, cs[i]);
          if (a.ng == 2) ct[i] = fmaf(At[ty * 4 + i][kk], btv, ct[i]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      Zs[r][tx] = cs[i];
      if (a.ng == 2) {
        Zt[r][tx] = ct[i];
      } else {
        float z = 0.f;
        if (m0 + r < N && v0 + tx < a.V) {
          const long long tr = a.teacher_rows ? a.teacher_rows[m0 + r] : (m0 + r);
          z = a.teacher[tr * a.teacher_pitch + v0 + tx];
        }
        Zt[r][tx] = z;
      }
    }
    __syncthreads();
    if (tid < TB) {
      const int r = tid;
      if (!DZ) {
        float cm_s = -INFINITY, cm_t = -INFINITY;
        for (int j = 0; j < TB && v0 + j < a.V; ++j) {
          cm_s = fmaxf(cm_s, Zs[r][j]);
          cm_t = fmaxf(cm_t, Zt[r][j]);
        }
        const float nm_s = fmaxf(m_s, cm_s), nm_t = fmaxf(m_t, cm_t);
        const float sc_s = ex2((m_s - nm_s) * kLog2e), sc_t = ex2((m_t - nm_t) * kLog2e);
        S_s *= sc_s;
        A *= sc_s;
        Bz *= sc_s;
        S_t *= sc_t;
        m_s = nm_s;
        m_t = nm_t;
        for (int j = 0; j < TB && v0 + j < a.V; ++j) {
          const float e = ex2(fmaf(Zs[r][j], kLog2e, -m_s * kLog2e));
          const float f = ex2(fmaf(Zt[r][j], kLog2e, -m_t * kLog2e));
          S_s += e;
          S_t += f;
          A = fmaf(e, Zs[r][j] - Zt[r][j], A);
          Bz = fmaf(e, Zs[r][j], Bz);
        }
        const unsigned d = static_cast<unsigned>(tgt - v0);
        if (tgt >= 0 && d < static_cast<unsigned>(TB)) a.tlogit[m0 + r] = Zs[r][d];
      } else if (m0 + r < N) {
        const float lse2 = a.rowc[m0 + r], cst = a.rowc[a.n_pad + m0 + r], g = a.rowc[2 * a.n_pad + m0 + r];
        float* out = a.dz + static_cast<long long>(m0 + r) * a.cw + (v0 - a.chunk_v0);
        for (int j = 0; j < TB && v0 - a.chunk_v0 + j < a.cw; ++j) {
          const float p = ex2(fmaf(Zs[r][j], kLog2e, -lse2));
          out[j] = g * p * ((Zs[r][j] - Zt[r][j]) + cst);
        }
      }
    }
    __syncthreads();
  }
  if (!DZ && tid < TB && u1 > u0) {
    float* base = a.part + static_cast<size_t>(split) * kStatVals * a.n_pad + (u0 / a.IT) * TB + tid;
    base[0] = m_s;
    base[a.n_pad] = S_s;
    base[2 * a.n_pad] = A;
    base[3 * a.n_pad] = m_t;
    base[4 * a.n_pad] = S_t;
    base[5 * a.n_pad] = Bz;
  }
}

// C[M, Nc] (+)= A B with arbitrary strides; 64x64 tiles, 4x4 per thread.
__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A, long long sam, long long sak,
                                                        const float* __restrict__ B, long long sbk, long long sbn,
                                                        float* __restrict__ C, long long ldc, int M, int Nc, int K,
                                                        int accumulate, const int32_t* __restrict__ n_dev,
                                                        int live_dim) {
  __shared__ float as[16][64 + 1], bs[16][64 + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (live_dim == 1) M = live_rows(n_dev, M);
  if (live_dim == 2) K = live_rows(n_dev, K);
  if (m0 >= M) return;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = tid; e < 16 * 64; e += 256) {
      const int kk = e / 64, i = e % 64;
      as[kk][i] = (m0 + i < M && k0 + kk < K) ? A[(m0 + i) * sam + (k0 + kk) * sak] : 0.f;
      bs[kk][i] = (n0 + i < Nc && k0 + kk < K) ? B[(k0 + kk) * sbk + (n0 + i) * sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(as[kk][ty * 4 + i], bs[kk][tx * 4 + j], acc[i][j]);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < Nc) {
        float* c = C + m * ldc + n;
        *c = accumulate ? *c + acc[i][j] : acc[i][j];
      }
    }
}

}  // namespace

cudaError_t launch_simt_fused(bool dz, const SimtArgs& a, dim3 grid, cudaStream_t s) {
  LaunchScope scope(dz ? K_DZ_SIMT : K_FWD_SIMT, s);
  if (dz)
    simt_fused_kernel<true><<<grid, 256, 0, s>>>(a);
  else
    simt_fused_kernel<false><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_simt_gemm(const float* A, long long sam, long long sak, const float* B, long long sbk,
                             long long sbn, float* C, long long ldc, int M, int Nc, int K, int accumulate,
                             const int32_t* n_dev, int live_dim, cudaStream_t s) {
  LaunchScope scope(K_GRAD_SIMT, s);
  dim3 grid((Nc + 63) / 64, (M + 63) / 64);
  simt_gemm_kernel<<<grid, 256, 0, s>>>(A, sam, sak, B, sbk, sbn, C, ldc, M, Nc, K, accumulate, n_dev, live_dim);
  return cudaGetLastError();
}

}  // namespace rkl
