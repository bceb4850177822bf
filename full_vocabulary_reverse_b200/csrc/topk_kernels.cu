// topk_kernels.cu -- the top-k estimator with both sides given as [T, V]
// logits: support selection, estimate and its gradient, bandwidth bound.
//
// "feat(mopd): add full-vocabulary on-policy distillation" (NeMo RL PR #3978),
// description: the exact full-vocabulary reverse KL is the K = V limit of the
// top-k MOPD estimator, whose score-function tail term vanishes when the
// support spans the vocabulary.  Reading used here (the page does not write
// the estimator out):
//   S      = the k largest student logits of the row, lower token id first
//            among equal logits;
//   L_hat  = sum_{v in S} p_s(v) w(v) + [y not in S] w(y),
//            w = log p_s - log p_t, y = the row's sampled (target) token;
//   dz(v)  = g (p_s(v) ([v in S](w(v) + 1) - C) + [v = y] a),
//            a = [y not in S](w(y) + 1), C = L_S + P_S + a,
//            L_S = sum_S p_s w, P_S = sum_S p_s.
//
// Forward, one CTA per trainable row:
//   pass A  streams z_s and z_t once: online log-sum-exp of both sides and a
//           256-bin histogram of the top byte of an order-preserving integer
//           key of z_s;
//   pass B  (one per further key byte: 1 for bf16, 3 for fp32) histograms the
//           next byte among the elements whose key matches the bytes chosen
//           so far; after the last level the key K* of the k-th largest
//           logit and the number r of elements of key K* that S takes are
//           known exactly (radix select);
//   pass C  streams z_s in index order, 2048 (bf16) or 1024 (fp32) elements
//           per round: elements of key > K* are in S, and elements of key
//           K* are ranked in index order by a block scan so that the first r
//           join S (this fixes v_last, the last of them); z_t is read only at
//           the members of S, which give L_S and P_S.
// Backward, one CTA per token row: dz_s in one stream over z_s and z_t, S
// decided by (key > K*) or (key = K* and v <= v_last), exact zero rows at
// masked positions.
#include <cuda_bf16.h>

#include <climits>

#include "kernels.h"
#include "sm100.cuh"

namespace rkl {
namespace {

constexpr int kTkThreads = 256;

__device__ __forceinline__ uint4 tk_ldg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Order-preserving unsigned key of a float: a < b  <=>  key(a) < key(b) for
// non-NaN values, and -0 and +0 share one key (they are equal logits).  For a
// bf16 value only the top 16 bits carry information (the kernels mask the low
// half, which is all ones for negative values).
__device__ __forceinline__ uint32_t fkey_raw(float x) {
  const uint32_t u = x == 0.f ? 0u : __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
struct TkIo;

template <>
struct TkIo<__nv_bfloat16> {
  static constexpr int VEC = 8;
  static constexpr int LEVELS = 2;  // a bf16 value has 16 significant key bits
  static constexpr uint32_t KMASK = 0xFFFF0000u;
  __device__ static void unpack(const uint4& w, float* out) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(a[i] << 16);
      out[2 * i + 1] = __uint_as_float(a[i] & 0xFFFF0000u);
    }
  }
  __device__ static float one(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }
  __device__ static uint4 pack(const float* d) {
    return make_uint4(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]), pack_bf16x2(d[4], d[5]),
                      pack_bf16x2(d[6], d[7]));
  }
  __device__ static __nv_bfloat16 cvt(float x) { return __float2bfloat16_rn(x); }
};

template <>
struct TkIo<float> {
  static constexpr int VEC = 4;
  static constexpr int LEVELS = 4;
  static constexpr uint32_t KMASK = 0xFFFFFFFFu;
  __device__ static void unpack(const uint4& w, float* out) {
    out[0] = __uint_as_float(w.x);
    out[1] = __uint_as_float(w.y);
    out[2] = __uint_as_float(w.z);
    out[3] = __uint_as_float(w.w);
  }
  __device__ static float one(const float* p, long long i) { return p[i]; }
  __device__ static uint4 pack(const float* d) {
    return make_uint4(__float_as_uint(d[0]), __float_as_uint(d[1]), __float_as_uint(d[2]), __float_as_uint(d[3]));
  }
  __device__ static float cvt(float x) { return x; }
};

struct Lse2 {
  float m_s, S_s, m_t, S_t;
};

__device__ __forceinline__ void lse_add(float& m, float& S, float x) {
  if (x > m) {
    S = S * ex2((m - x) * kLog2e) + 1.f;
    m = x;
  } else {
    S += ex2((x - m) * kLog2e);
  }
}

__device__ __forceinline__ void lse_join(float& m, float& S, float m2, float S2) {
  const float nm = fmaxf(m, m2);
  if (nm == -INFINITY) return;
  S = S * ex2((m - nm) * kLog2e) + S2 * ex2((m2 - nm) * kLog2e);
  m = nm;
}

// Block-wide inclusive sum of one int per thread (256 threads); returns the
// inclusive prefix of this thread and writes the block total to *total.
__device__ __forceinline__ int block_incl_scan(int x, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kTkThreads / 32 ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kTkThreads / 32) sh[lane] = w;
  }
  __syncthreads();
  const int r = x + (warp ? sh[warp - 1] : 0);
  *total = sh[kTkThreads / 32 - 1];
  __syncthreads();
  return r;
}

// Picks the histogram bin holding the need-th largest key (need >= 1, at most
// the histogram total): bins are scanned from the top.  Thread 0 only.
__device__ __forceinline__ void pick_bin(const int* hist, int need, int* bin, int* above) {
  int acc = 0;
  int b = 255;
  for (; b > 0; --b) {
    if (acc + hist[b] >= need) break;
    acc += hist[b];
  }
  *bin = b;
  *above = acc;
}

template <typename T>
__global__ void __launch_bounds__(kTkThreads) topk_fwd_kernel(const T* __restrict__ zs_all,
                                                              const T* __restrict__ zt_all,
                                                              const int32_t* __restrict__ row_idx,
                                                              const int32_t* __restrict__ targets, int N, int V,
                                                              long long k_sel, float* __restrict__ saved,
                                                              float* __restrict__ saved_tk) {
  using Io = TkIo<T>;
  constexpr int VEC = Io::VEC;
  __shared__ int hist[256];
  __shared__ int scan_sh[32];
  __shared__ float red_sh[4][kTkThreads / 32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need, s_vlast;
  __shared__ float s_lse[2];

  const int kr = blockIdx.x;
  if (kr >= N) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long r = row_idx[kr];
  const T* zs = zs_all + r * V;
  const T* zt = zt_all + r * V;
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(zs) | reinterpret_cast<uintptr_t>(zt)) & 15) == 0;
  const int nvec = vec_ok ? V / VEC : 0;
  const uint4* vs = reinterpret_cast<const uint4*>(zs);
  const uint4* vt = reinterpret_cast<const uint4*>(zt);
  const bool select = k_sel > 0 && k_sel < V;  // else S is empty or the whole row

  for (int i = tid; i < 256; i += kTkThreads) hist[i] = 0;
  __syncthreads();

  // ---- pass A: both log-sum-exps and the top-byte histogram of z_s
  float m_s = -INFINITY, S_s = 0.f, m_t = -INFINITY, S_t = 0.f;
  for (int i = tid; i < nvec; i += kTkThreads) {
    float xs[VEC], xt[VEC];
    Io::unpack(tk_ldg_v4(vs + i), xs);
    Io::unpack(tk_ldg_v4(vt + i), xt);
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      lse_add(m_s, S_s, xs[j]);
      lse_add(m_t, S_t, xt[j]);
      if (select) atomicAdd(&hist[(Io::KMASK & fkey_raw(xs[j])) >> 24], 1);
    }
  }
  for (int v = nvec * VEC + tid; v < V; v += kTkThreads) {
    const float xs = Io::one(zs, v), xt = Io::one(zt, v);
    lse_add(m_s, S_s, xs);
    lse_add(m_t, S_t, xt);
    if (select) atomicAdd(&hist[(Io::KMASK & fkey_raw(xs)) >> 24], 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lse_join(m_s, S_s, __shfl_xor_sync(0xffffffffu, m_s, o), __shfl_xor_sync(0xffffffffu, S_s, o));
    lse_join(m_t, S_t, __shfl_xor_sync(0xffffffffu, m_t, o), __shfl_xor_sync(0xffffffffu, S_t, o));
  }
  if (lane == 0) {
    red_sh[0][warp] = m_s;
    red_sh[1][warp] = S_s;
    red_sh[2][warp] = m_t;
    red_sh[3][warp] = S_t;
  }
  __syncthreads();
  if (tid == 0) {
    float a = red_sh[0][0], b = red_sh[1][0], c = red_sh[2][0], d = red_sh[3][0];
    for (int w = 1; w < kTkThreads / 32; ++w) {
      lse_join(a, b, red_sh[0][w], red_sh[1][w]);
      lse_join(c, d, red_sh[2][w], red_sh[3][w]);
    }
    s_lse[0] = a + logf(b);
    s_lse[1] = c + logf(d);
    if (select) {
      int bin, above;
      pick_bin(hist, static_cast<int>(k_sel), &bin, &above);
      s_prefix = static_cast<uint32_t>(bin) << 24;
      s_need = static_cast<int>(k_sel) - above;
    } else {
      // empty support: a key above every value; whole row: key 0 and no index cap
      s_prefix = k_sel <= 0 ? 0xFFFFFFFFu : 0u;
      s_need = 0;
    }
  }
  __syncthreads();

  // ---- pass B: the remaining key bytes of the k-th largest logit
  if (select) {
    for (int level = 1; level < Io::LEVELS; ++level) {
      const int shift = 24 - 8 * level;
      const uint32_t hi_mask = 0xFFFFFFFFu << (shift + 8);
      const uint32_t prefix = s_prefix;
      for (int i = tid; i < 256; i += kTkThreads) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < nvec; i += kTkThreads) {
        float xs[VEC];
        Io::unpack(tk_ldg_v4(vs + i), xs);
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
          const uint32_t key = (Io::KMASK & fkey_raw(xs[j]));
          if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
      }
      for (int v = nvec * VEC + tid; v < V; v += kTkThreads) {
        const uint32_t key = (Io::KMASK & fkey_raw(Io::one(zs, v)));
        if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid == 0) {
        int bin, above;
        pick_bin(hist, s_need, &bin, &above);
        s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
        s_need -= above;
      }
      __syncthreads();
    }
  }
  // Keys of bf16 values keep only their top 16 bits (KMASK), so after the two
  // levels s_prefix is the full key K*.
  const uint32_t kstar = s_prefix;
  const int need = s_need;  // members of key K*, taken lowest index first
  const float lse_s = s_lse[0], lse_t = s_lse[1];

  // ---- pass C: tie ranks in index order, and the sums over S
  float L_S = 0.f, P_S = 0.f;
  int carry = 0;
  if (tid == 0) s_vlast = select ? -1 : (k_sel <= 0 ? -1 : INT_MAX);
  constexpr int CH = VEC * kTkThreads;
  for (int c0 = 0; c0 < V; c0 += CH) {
    const int v0 = c0 + tid * VEC;
    float xs[VEC];
    if (vec_ok && v0 + VEC <= V) {
      Io::unpack(tk_ldg_v4(zs + v0), xs);
    } else {
#pragma unroll
      for (int j = 0; j < VEC; ++j) xs[j] = v0 + j < V ? Io::one(zs, v0 + j) : -INFINITY;
    }
    uint32_t keys[VEC];
    int eq = 0;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      keys[j] = v0 + j < V ? (Io::KMASK & fkey_raw(xs[j])) : 0u;
      eq += (select && v0 + j < V && keys[j] == kstar) ? 1 : 0;
    }
    int total = 0;
    int rank = carry;
    if (select) {
      const int incl = block_incl_scan(eq, scan_sh, &total);
      rank = carry + incl - eq;
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const int v = v0 + j;
      if (v >= V) continue;
      bool in;
      if (select) {
        in = keys[j] > kstar;
        if (keys[j] == kstar) {
          in = rank < need;
          if (rank == need - 1) s_vlast = v;
          ++rank;
        }
      } else {
        in = k_sel > 0;
      }
      if (in) {
        const float ls = xs[j] - lse_s;
        const float p = ex2(ls * kLog2e);
        const float w = ls - (Io::one(zt, v) - lse_t);
        L_S = fmaf(p, w, L_S);
        P_S += p;
      }
    }
    carry += total;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    L_S += __shfl_xor_sync(0xffffffffu, L_S, o);
    P_S += __shfl_xor_sync(0xffffffffu, P_S, o);
  }
  __syncthreads();
  if (lane == 0) {
    red_sh[0][warp] = L_S;
    red_sh[1][warp] = P_S;
  }
  __syncthreads();
  if (tid == 0) {
    float ls = 0.f, ps = 0.f;
    for (int w = 0; w < kTkThreads / 32; ++w) {
      ls += red_sh[0][w];
      ps += red_sh[1][w];
    }
    const int vlast = s_vlast;
    const int y = targets[r];
    float Lh, a;
    if (y < 0 || y >= V) {
      Lh = __int_as_float(0x7fffffff);
      a = Lh;
    } else {
      const float zy = Io::one(zs, y);
      const uint32_t ky = (Io::KMASK & fkey_raw(zy));
      const bool y_in = ky > kstar || (ky == kstar && y <= vlast);
      const float wy = (zy - lse_s) - (Io::one(zt, y) - lse_t);
      Lh = ls + (y_in ? 0.f : wy);
      a = y_in ? 0.f : wy + 1.f;
    }
    saved[3 * kr + 0] = lse_s;
    saved[3 * kr + 1] = lse_t;
    saved[3 * kr + 2] = Lh;
    saved_tk[4 * kr + 0] = ls + ps + a;  // C
    saved_tk[4 * kr + 1] = a;
    saved_tk[4 * kr + 2] = __uint_as_float(kstar);
    saved_tk[4 * kr + 3] = __int_as_float(vlast);
  }
}

// dz[t, :] for every token row t (exact zeros at masked rows).
template <typename T>
__global__ void __launch_bounds__(kTkThreads) topk_bwd_kernel(const T* __restrict__ zs_all,
                                                              const T* __restrict__ zt_all,
                                                              const int32_t* __restrict__ row_idx,
                                                              const int32_t* __restrict__ targets, int N, int n_pad,
                                                              int V, const float* __restrict__ saved,
                                                              const float* __restrict__ saved_tk,
                                                              const float* __restrict__ rowc, T* __restrict__ dz_all) {
  using Io = TkIo<T>;
  constexpr int VEC = Io::VEC;
  const long long t = blockIdx.x;
  int lo = 0, hi = N;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(row_idx[mid]) < t)
      lo = mid + 1;
    else
      hi = mid;
  }
  const int kr = lo;
  const bool hit = kr < N && row_idx[kr] == t;
  const T* zs = zs_all + t * V;
  const T* zt = zt_all + t * V;
  T* dz = dz_all + t * V;
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(zs) | reinterpret_cast<uintptr_t>(zt) |
                        reinterpret_cast<uintptr_t>(dz)) & 15) == 0;
  const int nvec = vec_ok ? V / VEC : 0;
  uint4* vd = reinterpret_cast<uint4*>(dz);
  if (!hit) {
    for (int i = threadIdx.x; i < nvec; i += kTkThreads) vd[i] = make_uint4(0, 0, 0, 0);
    for (int v = nvec * VEC + threadIdx.x; v < V; v += kTkThreads) dz[v] = Io::cvt(0.f);
    return;
  }
  const float lse_s = saved[3 * kr], lse_t = saved[3 * kr + 1];
  const float C = saved_tk[4 * kr], a = saved_tk[4 * kr + 1];
  const uint32_t kstar = __float_as_uint(saved_tk[4 * kr + 2]);
  const int vlast = __float_as_int(saved_tk[4 * kr + 3]);
  const float g = rowc[2 * n_pad + kr];
  const int y = targets[t];
  const float ga = g * a;
  const uint4* vs = reinterpret_cast<const uint4*>(zs);
  const uint4* vt = reinterpret_cast<const uint4*>(zt);
  for (int i = threadIdx.x; i < nvec; i += kTkThreads) {
    float xs[VEC], xt[VEC], d[VEC];
    Io::unpack(tk_ldg_v4(vs + i), xs);
    Io::unpack(tk_ldg_v4(vt + i), xt);
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const int v = i * VEC + j;
      const float ls = xs[j] - lse_s;
      const float p = ex2(ls * kLog2e);
      const uint32_t key = (Io::KMASK & fkey_raw(xs[j]));
      const bool in = key > kstar || (key == kstar && v <= vlast);
      const float coef = (in ? (ls - (xt[j] - lse_t)) + 1.f : 0.f) - C;
      d[j] = g * p * coef + (v == y ? ga : 0.f);
    }
    vd[i] = Io::pack(d);
  }
  for (int v = nvec * VEC + threadIdx.x; v < V; v += kTkThreads) {
    const float xs = Io::one(zs, v), xt = Io::one(zt, v);
    const float ls = xs - lse_s;
    const float p = ex2(ls * kLog2e);
    const uint32_t key = (Io::KMASK & fkey_raw(xs));
    const bool in = key > kstar || (key == kstar && v <= vlast);
    const float coef = (in ? (ls - (xt - lse_t)) + 1.f : 0.f) - C;
    dz[v] = Io::cvt(g * p * coef + (v == y ? ga : 0.f));
  }
}

}  // namespace

cudaError_t launch_topk_fwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, int V, long long k, float* saved, float* saved_tk,
                            cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_TOPK_FWD, s);
  if (bf16)
    topk_fwd_kernel<__nv_bfloat16><<<N, kTkThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(zs),
                                                            static_cast<const __nv_bfloat16*>(zt), row_idx, targets,
                                                            N, V, k, saved, saved_tk);
  else
    topk_fwd_kernel<float><<<N, kTkThreads, 0, s>>>(static_cast<const float*>(zs), static_cast<const float*>(zt),
                                                    row_idx, targets, N, V, k, saved, saved_tk);
  return cudaGetLastError();
}

cudaError_t launch_topk_bwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, int n_pad, long long T, int V, const float* saved,
                            const float* saved_tk, const float* rowc, void* dz, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  LaunchScope scope(K_TOPK_BWD, s);
  if (bf16)
    topk_bwd_kernel<__nv_bfloat16><<<static_cast<unsigned>(T), kTkThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(zs), static_cast<const __nv_bfloat16*>(zt), row_idx, targets, N, n_pad, V,
        saved, saved_tk, rowc, static_cast<__nv_bfloat16*>(dz));
  else
    topk_bwd_kernel<float><<<static_cast<unsigned>(T), kTkThreads, 0, s>>>(
        static_cast<const float*>(zs), static_cast<const float*>(zt), row_idx, targets, N, n_pad, V, saved, saved_tk,
        rowc, static_cast<float*>(dz));
  return cudaGetLastError();
}

}  // namespace rkl
