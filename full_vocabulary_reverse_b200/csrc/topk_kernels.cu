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
// Forward, one CTA per trainable row (256 threads, at most 40 registers so
// that six CTAs share an SM):
//   Threshold path (k <= 256, every thread owning logits).  z_s and z_t
//   stream once for both log-sum-exps, two 16-byte vectors of each per step.
//   After a first slice of the row, the k-th largest of the 256 threads'
//   running maxima, tau, bounds the k-th largest logit from below (k distinct
//   logits reach it).  The slice is read a second time and the rest
//   of the row as it streams, listing the logits whose keys reach tau
//   (key, token id) in shared memory.  The slice is sized for ~256 entries
//   on i.i.d. logits.
//   Histogram path (k > 256).  Pass A streams both rows for the log-sum-exps
//   and a 4096-bin histogram of the top 12 bits of an order-preserving key of
//   z_s; a block scan from the top finds the bin of the k-th largest key.
//   Pass B streams z_s again: keys above the bin are members of S (z_t is
//   gathered at them), keys in the bin are listed.
//   Either way a bitonic sort orders the list by key, lower token id first,
//   and its first r entries (r = k - members found before) complete S,
//   fixing the k-th key K* and v_last, the last token id of key K* taken.
//   If the list would exceed 4096 entries (long runs of tied logits), the
//   selection finishes exactly instead: radix passes over the key bits not
//   yet fixed give K*, and an index-ordered pass ranks the ties of key K* by
//   a block scan.
// Backward, one CTA per token row: dz_s in one stream over z_s and z_t, S
// decided by (key > K*) or (key = K* and v <= v_last), exact zero rows at
// masked positions.
#include <cuda_bf16.h>

#include <climits>
#include <type_traits>

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

// The forward's streaming loads bypass L1 (nothing it streams is reused
// from L1).
__device__ __forceinline__ uint4 tk_ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 tk_ldg_stream_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
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

// Keys of the two bf16 values packed in a 32-bit word, each in its half of the
// result (the same order-preserving map, applied to both halves at once).  A
// packed bf16 add of +0 turns -0 into +0 (a zero sum of opposite-signed zeros
// is +0 under round-to-nearest) and leaves every other value as it is; prmt
// with sign replication spreads each half's sign bit over the half; then a
// negative half is inverted and a positive one gets its sign bit set.
__device__ __forceinline__ uint32_t bf16_pair_keys(uint32_t w) {
  uint32_t c, s;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(w), "r"(0u));
  asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(s) : "r"(c));
  return c ^ (s | 0x80008000u);
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

constexpr int kTopShift = 20;            // first-level histogram: the top 12 key bits
constexpr int kTopBins = 1 << (32 - kTopShift);
constexpr int kCap = 4096;               // candidates sorted in shared memory
constexpr float kListTarget = 256.f;     // expected candidates on the threshold path

// Descending bitonic sort of n (a power of two, <= kCap) 64-bit entries in
// shared memory by the whole block.
__device__ __forceinline__ void bitonic_desc(unsigned long long* a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += kTkThreads) {
        const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));  // stride is a power of two
        const int hi = lo + stride;
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == ((lo & size) == 0)) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

// One student row's contribution to the sums over S: p_s(v) w(v) and p_s(v).
template <typename T>
__device__ __forceinline__ void add_member(float zs_v, const T* zt, int v, float lse_s, float lse_t, float& L_S,
                                           float& P_S) {
  const float ls = zs_v - lse_s;
  const float p = ex2(ls * kLog2e);
  L_S = fmaf(p, ls - (TkIo<T>::one(zt, v) - lse_t), L_S);
  P_S += p;
}

__device__ __forceinline__ void list_append(uint32_t key, int v, unsigned long long* cand, int* ncand) {
  const int slot = atomicAdd(ncand, 1);
  if (slot < kCap) cand[slot] = (static_cast<unsigned long long>(key) << 32) | (~static_cast<uint32_t>(v));
}

// Histogram path, pass B's decision for one logit (key, value x, token id v):
// keys above the bin are members, keys in the bin are candidates.
template <typename TT>
__device__ __forceinline__ void classify(uint32_t key, float x, int v, uint32_t bin, const TT* zt, float lse_s,
                                         float lse_t, float& L_S, float& P_S, unsigned long long* cand,
                                         int* ncand) {
  const uint32_t kb = key >> kTopShift;
  if (kb > bin) add_member<TT>(x, zt, v, lse_s, lse_t, L_S, P_S);
  if (kb == bin) list_append(key, v, cand, ncand);
}

// Threshold path: the logits of one vector of z_s (token ids v0, v0 + 1, ...)
// whose keys reach the bound tau go to the candidate list.
template <typename T>
__device__ __forceinline__ void list_vec(const uint4& ws, int v0, uint32_t tau, unsigned long long* cand,
                                         int* ncand) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // 16-bit keys sit in the top half: a low-half key reaches tau iff it is
    // >= tau >> 16, a high-half key iff the pair key is >= tau
    const uint32_t wz[4] = {ws.x, ws.y, ws.z, ws.w};
    uint32_t kp[4];
    bool any = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      kp[q] = bf16_pair_keys(wz[q]);
      any |= (kp[q] & 0xFFFFu) >= (tau >> 16) || kp[q] >= tau;
    }
    if (!any) return;  // the common case
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if ((kp[q] << 16) >= tau) list_append(kp[q] << 16, v0 + 2 * q, cand, ncand);
      if ((kp[q] & 0xFFFF0000u) >= tau) list_append(kp[q] & 0xFFFF0000u, v0 + 2 * q + 1, cand, ncand);
    }
  } else {
    float x[4];
    TkIo<float>::unpack(ws, x);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t key = fkey_raw(x[j]);
      if (key >= tau) list_append(key, v0 + j, cand, ncand);
    }
  }
}

// One vector of each row into the running log-sum-exps (maximum m, sum S of
// exp(x - m)).
template <int VEC>
__device__ __forceinline__ void lse_vec(const float* xs, const float* xt, float& m_s, float& S_s, float& m_t,
                                        float& S_t) {
  float cs = xs[0], ct = xt[0];
#pragma unroll
  for (int j = 1; j < VEC; ++j) {
    cs = fmaxf(cs, xs[j]);
    ct = fmaxf(ct, xt[j]);
  }
  if (cs > m_s) {
    S_s *= ex2((m_s - cs) * kLog2e);
    m_s = cs;
  }
  if (ct > m_t) {
    S_t *= ex2((m_t - ct) * kLog2e);
    m_t = ct;
  }
  const float ms2 = m_s * kLog2e, mt2 = m_t * kLog2e;
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    S_s += ex2(fmaf(xs[j], kLog2e, -ms2));
    S_t += ex2(fmaf(xt[j], kLog2e, -mt2));
  }
}

// The teacher values of one student vector (the VEC logits of type T from
// index i * VEC): one uint4 when both rows have the same type; for an fp32
// student row beside a bf16 teacher row, the four bf16 of one 8-byte load,
// widened exactly.
template <typename T, typename TT>
__device__ __forceinline__ void load_teacher_vec(const TT* zt, int i, float* out) {
  if constexpr (std::is_same<T, TT>::value) {
    TkIo<T>::unpack(tk_ldg_stream_v4(reinterpret_cast<const uint4*>(zt) + i), out);
  } else {
    static_assert(std::is_same<T, float>::value && std::is_same<TT, __nv_bfloat16>::value,
                  "mixed rows: fp32 student logits, bf16 teacher logits");
    const uint2 w = tk_ldg_stream_v2(reinterpret_cast<const uint2*>(zt) + i);
    out[0] = __uint_as_float(w.x << 16);
    out[1] = __uint_as_float(w.x & 0xFFFF0000u);
    out[2] = __uint_as_float(w.y << 16);
    out[3] = __uint_as_float(w.y & 0xFFFF0000u);
  }
}

// zs rows: block-local (local) or token rows; zt rows: block-local (t_local)
// or token rows, of type TT with pitch tpitch.  The teacher-logits payload
// pairs the block's fp32 student logits with the shipped bf16 teacher rows.
template <typename T, typename TT = T>
__global__ void __launch_bounds__(kTkThreads, 6) topk_fwd_kernel(const T* __restrict__ zs_all,
                                                              const TT* __restrict__ zt_all,
                                                              const int32_t* __restrict__ row_idx,
                                                              const int32_t* __restrict__ targets, int N,
                                                              const int32_t* __restrict__ n_dev, int n_base, int V,
                                                              long long k_sel, float* __restrict__ saved,
                                                              float* __restrict__ saved_tk, long long zpitch,
                                                              int local, long long tpitch, int t_local) {
  using Io = TkIo<T>;
  constexpr int VEC = Io::VEC;
  // 32 KB: the 4096-bin histogram of pass A (histogram path) or the sort of
  // the threads' maxima (threshold path), then the candidate list
  __shared__ unsigned long long buf[kCap];
  int* hist = reinterpret_cast<int*>(buf);
  __shared__ int hist2[256];
  __shared__ int scan_sh[32];
  __shared__ float red_sh[4][kTkThreads / 32];
  __shared__ uint32_t s_kstar, s_tau;
  __shared__ int s_need, s_vlast, s_ncand, s_bin;
  __shared__ float s_lse[2];

  const int kr = blockIdx.x;
  if (kr >= live_rows(n_dev, N, n_base)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long r = row_idx[kr];  // token position (sampled token)
  const long long zr = local ? kr : r;  // logit row: a block-local row, or the token position
  const T* zs = zs_all + zr * zpitch;
  const TT* zt = zt_all + (t_local ? kr : r) * tpitch;
  const bool vec_ok = (reinterpret_cast<uintptr_t>(zs) & 15) == 0 &&
                      (reinterpret_cast<uintptr_t>(zt) & (VEC * sizeof(TT) - 1)) == 0;
  const int nvec = vec_ok ? V / VEC : 0;
  const uint4* vs = reinterpret_cast<const uint4*>(zs);
  // 0: empty support, 1: the whole row, 2: a proper subset to select
  const int mode = k_sel <= 0 ? 0 : (k_sel >= V ? 1 : 2);
  // small k with every thread owning logits: the k-th largest of the
  // threads' maxima bounds the k-th largest logit from below, and no
  // histogram is needed
  const bool thr = mode == 2 && k_sel <= kTkThreads && nvec >= kTkThreads;

  if (mode == 2 && !thr)
    for (int i = tid; i < kTopBins; i += kTkThreads) hist[i] = 0;
  if (tid == 0) {
    s_ncand = 0;
    s_kstar = mode == 0 ? 0xFFFFFFFFu : 0u;  // above every key / below every key
    s_vlast = mode == 0 ? -1 : INT_MAX;
  }
  __syncthreads();

  // ---- pass A: both log-sum-exps, and the 12-bit histogram of the z_s keys
  // or (threshold path) the candidate list
  float m_s = -INFINITY, S_s = 0.f, m_t = -INFINITY, S_t = 0.f;
  // Threshold path: vectors [0, i1) stream by before the bound is known and
  // are read a second time to be listed; the rest of the row is listed as it
  // streams.  The bound is about the (1 - k/256) quantile
  // of a thread's maximum over its e logits of [0, i1), so about
  // V ln(256 / (256 - k)) / e logits reach it: e is sized for kListTarget.
  int i1 = nvec;
  if (thr) {
    const float e = static_cast<float>(V) * __logf(256.f / (256.5f - static_cast<float>(k_sel))) / kListTarget;
    const int j1 = max(1, static_cast<int>(ceilf(e / VEC)));
    i1 = j1 >= nvec / kTkThreads ? nvec : j1 * kTkThreads;
  }
  for (int i = tid; i < i1; i += kTkThreads) {
    float xs[VEC], xt[VEC];
    const uint4 ws = tk_ldg_stream_v4(vs + i);
    Io::unpack(ws, xs);
    load_teacher_vec<T, TT>(zt, i, xt);
    if (mode == 2 && !thr) {
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        const uint32_t wz[4] = {ws.x, ws.y, ws.z, ws.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t kp = bf16_pair_keys(wz[q]);
          atomicAdd(&hist[(kp >> (kTopShift - 16)) & (kTopBins - 1)], 1);
          atomicAdd(&hist[kp >> kTopShift], 1);
        }
      } else {
#pragma unroll
        for (int j = 0; j < VEC; ++j) atomicAdd(&hist[(Io::KMASK & fkey_raw(xs[j])) >> kTopShift], 1);
      }
    }
    lse_vec<VEC>(xs, xt, m_s, S_s, m_t, S_t);
  }
  uint32_t tau = 0u;
  if (thr) {
    // tau = the k-th largest of the threads' maximum keys so far: k distinct
    // logits reach it, so every logit of the row's top k does too
    buf[tid] = (static_cast<unsigned long long>(Io::KMASK & fkey_raw(m_s)) << 32) | tid;
    __syncthreads();
    bitonic_desc(buf, kTkThreads);
    if (tid == 0) {
      s_tau = static_cast<uint32_t>(buf[k_sel - 1] >> 32);
      s_need = static_cast<int>(k_sel);
    }
    __syncthreads();
    tau = s_tau;
    for (int i = tid; i < i1; i += kTkThreads) list_vec<T>(tk_ldg_stream_v4(vs + i), i * VEC, tau, buf, &s_ncand);
    int i = i1 + tid;
    // two vectors of each row per step, all four loads issued first
    for (; i + kTkThreads < nvec; i += 2 * kTkThreads) {
      if constexpr (std::is_same<T, TT>::value) {
        const uint4* vt = reinterpret_cast<const uint4*>(zt);
        const uint4 a0 = tk_ldg_stream_v4(vs + i), b0 = tk_ldg_stream_v4(vt + i);
        const uint4 a1 = tk_ldg_stream_v4(vs + i + kTkThreads), b1 = tk_ldg_stream_v4(vt + i + kTkThreads);
        float xs[VEC], xt[VEC];
        list_vec<T>(a0, i * VEC, tau, buf, &s_ncand);
        Io::unpack(a0, xs);
        Io::unpack(b0, xt);
        lse_vec<VEC>(xs, xt, m_s, S_s, m_t, S_t);
        list_vec<T>(a1, (i + kTkThreads) * VEC, tau, buf, &s_ncand);
        Io::unpack(a1, xs);
        Io::unpack(b1, xt);
        lse_vec<VEC>(xs, xt, m_s, S_s, m_t, S_t);
      } else {
        const uint4 a0 = tk_ldg_stream_v4(vs + i);
        const uint4 a1 = tk_ldg_stream_v4(vs + i + kTkThreads);
        float xs[VEC], xt[VEC], xt1[VEC];
        load_teacher_vec<T, TT>(zt, i, xt);
        load_teacher_vec<T, TT>(zt, i + kTkThreads, xt1);
        list_vec<T>(a0, i * VEC, tau, buf, &s_ncand);
        Io::unpack(a0, xs);
        lse_vec<VEC>(xs, xt, m_s, S_s, m_t, S_t);
        list_vec<T>(a1, (i + kTkThreads) * VEC, tau, buf, &s_ncand);
        Io::unpack(a1, xs);
        lse_vec<VEC>(xs, xt1, m_s, S_s, m_t, S_t);
      }
    }
    for (; i < nvec; i += kTkThreads) {
      float xs[VEC], xt[VEC];
      const uint4 ws = tk_ldg_stream_v4(vs + i);
      list_vec<T>(ws, i * VEC, tau, buf, &s_ncand);
      Io::unpack(ws, xs);
      load_teacher_vec<T, TT>(zt, i, xt);
      lse_vec<VEC>(xs, xt, m_s, S_s, m_t, S_t);
    }
  }
  for (int v = nvec * VEC + tid; v < V; v += kTkThreads) {
    const float xs = Io::one(zs, v), xt = TkIo<TT>::one(zt, v);
    lse_add(m_s, S_s, xs);
    lse_add(m_t, S_t, xt);
    if (mode == 2) {
      const uint32_t key = Io::KMASK & fkey_raw(xs);
      if (!thr)
        atomicAdd(&hist[key >> kTopShift], 1);
      else if (key >= tau)
        list_append(key, v, buf, &s_ncand);
    }
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
  }
  if (mode == 2 && !thr) {
    // the bin of the k-th largest key: thread tid owns bins [16 g, 16 g + 16),
    // g = 255 - tid, so an inclusive scan in thread order counts from the top
    constexpr int PER = kTopBins / kTkThreads;
    const int g = kTkThreads - 1 - tid;
    int sg = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) sg += hist[PER * g + j];
    int tot;
    const int incl = block_incl_scan(sg, scan_sh, &tot);
    const int above = incl - sg;
    if (above < k_sel && k_sel <= incl) {
      int acc = above;
      for (int j = PER - 1; j >= 0; --j) {
        const int bn = PER * g + j;
        if (acc + hist[bn] >= k_sel) {
          s_bin = bn;
          s_need = static_cast<int>(k_sel) - acc;
          break;
        }
        acc += hist[bn];
      }
    }
  }
  __syncthreads();
  const float lse_s = s_lse[0], lse_t = s_lse[1];
  float L_S = 0.f, P_S = 0.f;

  if (mode == 1) {
    // ---- the whole row is the support
    for (int i = tid; i < nvec; i += kTkThreads) {
      float xs[VEC], xt[VEC];
      Io::unpack(tk_ldg_stream_v4(vs + i), xs);
      load_teacher_vec<T, TT>(zt, i, xt);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        const float ls = xs[j] - lse_s;
        const float p = ex2(ls * kLog2e);
        L_S = fmaf(p, ls - (xt[j] - lse_t), L_S);
        P_S += p;
      }
    }
    for (int v = nvec * VEC + tid; v < V; v += kTkThreads) add_member<TT>(Io::one(zs, v), zt, v, lse_s, lse_t, L_S, P_S);
  } else if (mode == 2) {
    // ---- pass B (histogram path): keys above the bin are members, keys in
    // the bin are candidates; the threshold path has its list already
    const uint32_t bin = static_cast<uint32_t>(s_bin);
    const int need = s_need;
    if (!thr) {
      // 16-bit (bf16) keys sit in the top half: a low-half key is in a bin
      // >= bin iff it is >= bin << 4, a high-half key iff the pair key is
      // >= bin << 20
      const uint32_t lo_thr = bin << (kTopShift - 16), hi_thr = bin << kTopShift;
      for (int i = tid; i < nvec; i += kTkThreads) {
        float xs[VEC];
        const uint4 ws = tk_ldg_stream_v4(vs + i);
        uint32_t keys[VEC];
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
          const uint32_t wz[4] = {ws.x, ws.y, ws.z, ws.w};
          uint32_t kp[4];
          bool any = false;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            kp[q] = bf16_pair_keys(wz[q]);
            any |= (kp[q] & 0xFFFFu) >= lo_thr || kp[q] >= hi_thr;
          }
          if (!any) continue;  // no key of these 8 reaches the bin (the common case)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            keys[2 * q] = kp[q] << 16;
            keys[2 * q + 1] = kp[q] & 0xFFFF0000u;
          }
          Io::unpack(ws, xs);
        } else {
          Io::unpack(ws, xs);
#pragma unroll
          for (int j = 0; j < VEC; ++j) keys[j] = Io::KMASK & fkey_raw(xs[j]);
        }
#pragma unroll
        for (int j = 0; j < VEC; ++j)
          classify<TT>(keys[j], xs[j], i * VEC + j, bin, zt, lse_s, lse_t, L_S, P_S, buf, &s_ncand);
      }
      for (int v = nvec * VEC + tid; v < V; v += kTkThreads) {
        const float x = Io::one(zs, v);
        classify<TT>(Io::KMASK & fkey_raw(x), x, v, bin, zt, lse_s, lse_t, L_S, P_S, buf, &s_ncand);
      }
    }
    __syncthreads();
    const int nc = s_ncand;
    if (nc <= kCap) {
      // ---- the candidates in key order (lower token id first on equal keys);
      // the first `need` of them complete the support
      int n2 = 2;
      while (n2 < nc) n2 <<= 1;
      for (int i = nc + tid; i < n2; i += kTkThreads) buf[i] = 0ull;
      __syncthreads();
      bitonic_desc(buf, n2);
      for (int j = tid; j < need; j += kTkThreads) {
        const int v = static_cast<int>(~static_cast<uint32_t>(buf[j]));
        add_member<TT>(Io::one(zs, v), zt, v, lse_s, lse_t, L_S, P_S);
      }
      if (tid == 0) {
        const unsigned long long e = buf[need - 1];
        s_kstar = static_cast<uint32_t>(e >> 32);
        s_vlast = static_cast<int>(~static_cast<uint32_t>(e));
      }
    } else {
      // ---- too many candidates: a radix select over the key bits below the
      // ones already fixed (the bin's 12, or none on the threshold path) gives
      // K*, then the ties of key K* are ranked in index order.  Keys whose
      // fixed bits are above the prefix are members added in pass B.
      const int lo_end = Io::KMASK == 0xFFFF0000u ? 16 : 0;
      const int hi0 = thr ? 32 : kTopShift;
      const uint32_t fixed = thr ? 0u : ~0u << kTopShift;  // the key bits fixed before the radix passes
      const uint32_t prefix0 = thr ? 0u : bin << kTopShift;
      uint32_t prefix = prefix0;
      int rem = need;
      for (int hi = hi0; hi > lo_end;) {
        const int width = hi - lo_end < 8 ? hi - lo_end : 8;
        const int sh = hi - width;
        const uint32_t hmask = hi >= 32 ? 0u : ~0u << hi;
        for (int i = tid; i < 256; i += kTkThreads) hist2[i] = 0;
        __syncthreads();
        for (int v = tid; v < V; v += kTkThreads) {
          const uint32_t key = Io::KMASK & fkey_raw(Io::one(zs, v));
          if ((key & hmask) == (prefix & hmask)) atomicAdd(&hist2[(key >> sh) & ((1u << width) - 1u)], 1);
        }
        __syncthreads();
        if (tid == 0) {
          int bn, ab;
          pick_bin(hist2, rem, &bn, &ab);
          s_bin = bn;
          s_need = rem - ab;
        }
        __syncthreads();
        prefix |= static_cast<uint32_t>(s_bin) << sh;
        rem = s_need;
        hi = sh;
        __syncthreads();
      }
      const uint32_t kstar = prefix;
      int carry = 0;
      constexpr int CH = VEC * kTkThreads;
      for (int c0 = 0; c0 < V; c0 += CH) {
        const int v0 = c0 + tid * VEC;
        float xs[VEC];
        uint32_t keys[VEC];
        int eq = 0;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
          xs[j] = v0 + j < V ? Io::one(zs, v0 + j) : -INFINITY;
          keys[j] = v0 + j < V ? (Io::KMASK & fkey_raw(xs[j])) : 0u;
          eq += (v0 + j < V && keys[j] == kstar) ? 1 : 0;
        }
        int total;
        const int incl = block_incl_scan(eq, scan_sh, &total);
        int rank = carry + incl - eq;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
          const int v = v0 + j;
          if (v >= V || (keys[j] & fixed) != prefix0) continue;  // members added in pass B, or below
          bool in = keys[j] > kstar;
          if (keys[j] == kstar) {
            in = rank < rem;
            if (rank == rem - 1) s_vlast = v;
            ++rank;
          }
          if (in) add_member<TT>(xs[j], zt, v, lse_s, lse_t, L_S, P_S);
        }
        carry += total;
      }
      if (tid == 0) s_kstar = kstar;
    }
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
    const uint32_t kstar = s_kstar;
    const int vlast = s_vlast;
    const int y = targets[r];
    float Lh, a;
    if (y < 0 || y >= V) {
      Lh = __int_as_float(0x7fffffff);
      a = Lh;
    } else {
      const float zy = Io::one(zs, y);
      const uint32_t ky = Io::KMASK & fkey_raw(zy);
      const bool y_in = ky > kstar || (ky == kstar && y <= vlast);
      const float wy = (zy - lse_s) - (TkIo<TT>::one(zt, y) - lse_t);
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
                                                              const int32_t* __restrict__ targets, int N,
                                                              const int32_t* __restrict__ n_dev, int n_pad,
                                                              int V, const float* __restrict__ saved,
                                                              const float* __restrict__ saved_tk,
                                                              const float* __restrict__ rowc, T* __restrict__ dz_all) {
  using Io = TkIo<T>;
  constexpr int VEC = Io::VEC;
  const long long t = blockIdx.x;
  N = live_rows(n_dev, N);
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

// Per-row constants of the hidden-payload top-k dz pass, [6][n_pad]:
// lse_t - lse_s, C, a, and the bit patterns of K*, v_last and the sampled
// token id; padding rows get values that select nothing.
__global__ void __launch_bounds__(256) topk_rowk_kernel(const float* __restrict__ saved,
                                                        const float* __restrict__ saved_tk,
                                                        const int32_t* __restrict__ row_idx,
                                                        const int32_t* __restrict__ targets, int N,
                                                        const int32_t* __restrict__ n_dev, int n_pad,
                                                        float* __restrict__ rowk) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_pad) return;
  N = live_rows(n_dev, N);
  float v[6] = {0.f, 0.f, 0.f, __uint_as_float(0xFFFFFFFFu), __int_as_float(-1), __int_as_float(-1)};
  if (p < N) {
    v[0] = saved[3 * p + 1] - saved[3 * p];
    v[1] = saved_tk[4 * p];
    v[2] = saved_tk[4 * p + 1];
    v[3] = saved_tk[4 * p + 2];
    v[4] = saved_tk[4 * p + 3];
    v[5] = __int_as_float(targets[row_idx[p]]);
  }
#pragma unroll
  for (int i = 0; i < 6; ++i) rowk[static_cast<size_t>(i) * n_pad + p] = v[i];
}

}  // namespace

cudaError_t launch_topk_fwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, const int32_t* n_dev, int n_base, int V, long long k,
                            float* saved, float* saved_tk, long long zpitch, bool local, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_TOPK_FWD, s);
  if (bf16)
    topk_fwd_kernel<__nv_bfloat16><<<N, kTkThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(zs),
                                                            static_cast<const __nv_bfloat16*>(zt), row_idx, targets,
                                                            N, n_dev, n_base, V, k, saved, saved_tk, zpitch,
                                                            local ? 1 : 0, zpitch, local ? 1 : 0);
  else
    topk_fwd_kernel<float><<<N, kTkThreads, 0, s>>>(static_cast<const float*>(zs), static_cast<const float*>(zt),
                                                    row_idx, targets, N, n_dev, n_base, V, k, saved, saved_tk, zpitch,
                                                    local ? 1 : 0, zpitch, local ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_topk_fwd_tlogits(const float* zs, const uint16_t* teacher, long long tpitch,
                                    const int32_t* row_idx, const int32_t* targets, int N, const int32_t* n_dev,
                                    int n_base, int V, long long k, float* saved, float* saved_tk, long long zpitch,
                                    cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_TOPK_FWD, s);
  topk_fwd_kernel<float, __nv_bfloat16><<<N, kTkThreads, 0, s>>>(
      zs, reinterpret_cast<const __nv_bfloat16*>(teacher), row_idx, targets, N, n_dev, n_base, V, k, saved, saved_tk,
      zpitch, 1, tpitch, 0);
  return cudaGetLastError();
}

cudaError_t launch_topk_rowk(const float* saved, const float* saved_tk, const int32_t* row_idx,
                             const int32_t* targets, int N, const int32_t* n_dev, int n_pad, float* rowk,
                             cudaStream_t s) {
  LaunchScope scope(K_TOPK_ROWK, s);
  topk_rowk_kernel<<<(n_pad + 255) / 256, 256, 0, s>>>(saved, saved_tk, row_idx, targets, N, n_dev, n_pad, rowk);
  return cudaGetLastError();
}

cudaError_t launch_topk_bwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx,
                            const int32_t* targets, int N, const int32_t* n_dev, int n_pad, long long T, int V,
                            const float* saved, const float* saved_tk, const float* rowc, void* dz, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  LaunchScope scope(K_TOPK_BWD, s);
  if (bf16)
    topk_bwd_kernel<__nv_bfloat16><<<static_cast<unsigned>(T), kTkThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(zs), static_cast<const __nv_bfloat16*>(zt), row_idx, targets, N, n_dev,
        n_pad, V, saved, saved_tk, rowc, static_cast<__nv_bfloat16*>(dz));
  else
    topk_bwd_kernel<float><<<static_cast<unsigned>(T), kTkThreads, 0, s>>>(
        static_cast<const float*>(zs), static_cast<const float*>(zt), row_idx, targets, N, n_dev, n_pad, V, saved,
        saved_tk, rowc, static_cast<float*>(dz));
  return cudaGetLastError();
}

}  // namespace rkl
