// small_kernels.cu -- the bandwidth-bound and bookkeeping steps of the loss:
//   S1 compaction of the trainable rows, S2 row gather, S8 teacher
//   log-sum-exp over shipped logits, S4 split merge / scatter / reduction,
//   S5 per-row backward weights, and the final dH scatter.
// Sources: "fix(megatron): compact actor logits before projection" (slime PR
// #2310, Summary: project only the N loss-masked rows, scatter scalars back,
// empty masks keep zero gradients) and "feat(mopd): add full-vocabulary
// on-policy distillation" (NeMo RL PR #3978: the objective, the logits
// payload, the token-level / nested per-sequence reduction).
#include <cuda_bf16.h>

#include <cfloat>

#include "bounds.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rkl {
RKL_DEFINE_BOUNDS_READER(read_and_clear_bounds_small)

namespace {

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, long long key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(a[mid]) < key)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

// --------------------------------------------------------------------- S1
// One CTA, 1024 threads; tiles of 8 mask bytes per thread; block-wide
// exclusive scan; ascending row indices by construction.
__global__ void __launch_bounds__(1024) compact_kernel(const uint8_t* __restrict__ mask, long long T,
                                                       int32_t* __restrict__ row_idx, int32_t* __restrict__ n_dev) {
  constexpr int ITEMS = 8;
  __shared__ int warp_incl[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (long long base = 0; base < T; base += 1024LL * ITEMS) {
    const long long i0 = base + static_cast<long long>(tid) * ITEMS;
    int flags = 0, cnt = 0;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
      const bool f = (i0 + k < T) && mask[i0 + k] != 0;
      flags |= static_cast<int>(f) << k;
      cnt += f;
    }
    int x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_incl[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_incl[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_incl[lane] = w;
    }
    __syncthreads();
    int pos = carry + (warp ? warp_incl[warp - 1] : 0) + x - cnt;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k)
      if (flags & (1 << k)) row_idx[pos++] = static_cast<int32_t>(i0 + k);
    __syncthreads();
    if (tid == 0) carry += warp_incl[31];
    __syncthreads();
  }
  if (tid == 0) *n_dev = carry;
}

// --------------------------------------------------------------------- S2
// hc[p] = h[row_idx[k]] for p < n_rows, k = slot_k[p] (or p without a slot
// map); a slot with k < 0 (padding between teacher groups) becomes a zero
// row.  With a device row count n, rows [n, n rounded up to 256) -- the rest
// of the last pair tile, which the tensor-core kernels read -- become zero
// rows too.  blockIdx.y selects student / teacher.
__global__ void __launch_bounds__(256) gather_kernel(const uint8_t* __restrict__ h_s, const uint8_t* __restrict__ h_t,
                                                     uint8_t* __restrict__ hc_s, uint8_t* __restrict__ hc_t,
                                                     const int32_t* __restrict__ row_idx,
                                                     const int32_t* __restrict__ slot_k, int n_rows,
                                                     const int32_t* __restrict__ n_dev, int row_bytes, long long T) {
  const uint8_t* src = blockIdx.y == 0 ? h_s : h_t;
  uint8_t* dst = blockIdx.y == 0 ? hc_s : hc_t;
  const int n_live = live_rows(n_dev, n_rows);
  const int n_end = n_dev ? ((n_live + 2 * kBM - 1) / (2 * kBM)) * (2 * kBM) : n_rows;
  for (int p = blockIdx.x; p < n_end; p += gridDim.x) {
    int k = p < n_live ? (slot_k ? slot_k[p] : p) : -1;
    if (k >= 0 && !RKL_BOUNDS(row_idx[k] >= 0 && row_idx[k] < T)) k = -1;  // (debug build) a zero row instead
    uint8_t* d = dst + static_cast<long long>(p) * row_bytes;
    if (k < 0) {
      for (int i = threadIdx.x; i < row_bytes / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(d)[i] = 0u;
      continue;
    }
    const uint8_t* s = src + static_cast<long long>(row_idx[k]) * row_bytes;
    if ((row_bytes & 15) == 0) {
      const uint4* s4 = reinterpret_cast<const uint4*>(s);
      uint4* d4 = reinterpret_cast<uint4*>(d);
      for (int i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) d4[i] = __ldg(s4 + i);
    } else {
      const uint32_t* s1 = reinterpret_cast<const uint32_t*>(s);
      uint32_t* d1 = reinterpret_cast<uint32_t*>(d);
      for (int i = threadIdx.x; i < row_bytes / 4; i += blockDim.x) d1[i] = __ldg(s1 + i);
    }
  }
}

// --------------------------------------------------------------------- S8
// lse_t[k] = log sum_v exp(z_t[row_idx[k], v]) over the shipped teacher
// logits.  One CTA per row, 16-byte streaming loads, four in flight per
// thread, per-thread online (max, sum), then a block merge.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float nm = fmaxf(m, m2);
  if (nm == -INFINITY) return;
  s = s * ex2((m - nm) * kLog2e) + s2 * ex2((m2 - nm) * kLog2e);
  m = nm;
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T>
__device__ __forceinline__ void vec_to_float(const uint4& w, float* out);

template <>
__device__ __forceinline__ void vec_to_float<__nv_bfloat16>(const uint4& w, float* out) {
  const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(a[i] << 16);
    out[2 * i + 1] = __uint_as_float(a[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void vec_to_float<float>(const uint4& w, float* out) {
  out[0] = __uint_as_float(w.x);
  out[1] = __uint_as_float(w.y);
  out[2] = __uint_as_float(w.z);
  out[3] = __uint_as_float(w.w);
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__global__ void __launch_bounds__(256) teacher_lse_kernel(const T* __restrict__ logits,
                                                          const int32_t* __restrict__ row_idx, int N,
                                                          const int32_t* __restrict__ n_dev, int V, long long pitch,
                                                          float* __restrict__ lse_t, long long rows) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int UNROLL = 4;
  const int k = blockIdx.x;
  if (k >= live_rows(n_dev, N)) return;
  const long long r = row_idx ? row_idx[k] : k;
  if (!RKL_BOUNDS(r >= 0 && r < rows)) return;
  const T* row = logits + r * pitch;
  float m = -INFINITY, s = 0.f;
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
  int done = 0;
  if (vec_ok) {
    const int nvec = V / VEC;
    const uint4* rv = reinterpret_cast<const uint4*>(row);
    int i = threadIdx.x;
    for (; i + (UNROLL - 1) * 256 < nvec; i += UNROLL * 256) {
      uint4 w[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) w[u] = ldg_stream_v4(rv + i + u * 256);
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        float x[VEC];
        vec_to_float<T>(w[u], x);
        float vm = x[0];
#pragma unroll
        for (int j = 1; j < VEC; ++j) vm = fmaxf(vm, x[j]);
        if (vm > m) {
          s *= ex2((m - vm) * kLog2e);
          m = vm;
        }
        const float m2 = m * kLog2e;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc += ex2(fmaf(x[j], kLog2e, -m2));
        s += acc;
      }
    }
    for (; i < nvec; i += 256) {
      float x[VEC];
      vec_to_float<T>(ldg_stream_v4(rv + i), x);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        if (x[j] > m) {
          s *= ex2((m - x[j]) * kLog2e);
          m = x[j];
        }
        s += ex2((x[j] - m) * kLog2e);
      }
    }
    done = nvec * VEC;
  }
  for (int v = done + threadIdx.x; v < V; v += 256) {
    const float x = to_f<T>(row[v]);
    if (x > m) {
      s *= ex2((m - x) * kLog2e);
      m = x;
    }
    s += ex2((x - m) * kLog2e);
  }
  // block merge (fixed order)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, m2, s2);
  }
  __shared__ float sm[8], ss[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sm[warp] = m;
    ss[warp] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = sm[0], Ssum = ss[0];
    for (int w = 1; w < 8; ++w) lse_merge(M, Ssum, sm[w], ss[w]);
    lse_t[k] = M + logf(Ssum);
  }
}

// --------------------------------------------------------------------- S4
// Merge the per-slot statistics of each row; L = A/S_s - lse_s + lse_t.
// A block takes 32 consecutive rows (lane = row) and its 8 warps split the
// slots into 8 contiguous ranges, so every load of a warp reads 32
// consecutive rows of one slot (coalesced) and each warp has few slots to
// chain.  Within a warp the slots are taken four at a time and merged by a
// fixed tree, ((g, g+1), (g+2, g+3)), into the running result; the 8
// partial results are then merged in warp order by warp 0.  The same order
// on every run.  Student and teacher statistics go through identical
// operations, so teacher == student gives L = 0 exactly.
struct Stat3 {
  float m, S, A, Bz;
};

__device__ __forceinline__ void merge3(Stat3& a, const Stat3& b) {
  const float nm = fmaxf(a.m, b.m);
  if (nm == -INFINITY) return;
  const float ea = expf(a.m - nm), eb = expf(b.m - nm);
  a.S = a.S * ea + b.S * eb;
  a.A = a.A * ea + b.A * eb;
  a.Bz = a.Bz * ea + b.Bz * eb;
  a.m = nm;
}

__device__ __forceinline__ void load_slot(const float* __restrict__ part, int g, int n_pad, int k, bool teacher,
                                          Stat3& s, Stat3& t) {
  const float* b = part + static_cast<size_t>(g) * kStatVals * n_pad + k;
  s = Stat3{b[0], b[n_pad], b[2 * n_pad], b[5 * n_pad]};
  t = teacher ? Stat3{b[3 * n_pad], b[4 * n_pad], 0.f, 0.f} : Stat3{-INFINITY, 0.f, 0.f, 0.f};
}

constexpr int kCombineWarps = 8;

// Optional student statistics of row k (nullable outputs): entropy
// lse_s - sum p_s z_s = lse_s - Bz / S_s, and target log-prob tlogit - lse_s.
// Statistics row k (a slot of the teacher-grouped layout when slot_k is
// given) is written to compact row out = slot_k[k]; padding slots are skipped.
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(
    const float* __restrict__ part, int S, int n_pad, int n_rows, const int32_t* __restrict__ n_dev,
    int teacher_from_part, const float* __restrict__ lse_ext, const float* __restrict__ tlogit,
    float* __restrict__ saved, float* __restrict__ ent_rows, float* __restrict__ lp_rows,
    const int32_t* __restrict__ slot_k) {
  __shared__ Stat3 sh_s[kCombineWarps][32], sh_t[kCombineWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = blockIdx.x * 32 + lane;
  const int n_live = live_rows(n_dev, n_rows);
  const bool teacher = teacher_from_part != 0;
  Stat3 s{-INFINITY, 0.f, 0.f, 0.f}, t{-INFINITY, 0.f, 0.f, 0.f};
  if (k < n_live) {
    const int g0 = static_cast<int>((static_cast<long long>(S) * warp) / kCombineWarps);
    const int g1 = static_cast<int>((static_cast<long long>(S) * (warp + 1)) / kCombineWarps);
    int g = g0;
    for (; g + 4 <= g1; g += 4) {
      Stat3 s0, t0, s1, t1, s2, t2, s3, t3;
      load_slot(part, g, n_pad, k, teacher, s0, t0);
      load_slot(part, g + 1, n_pad, k, teacher, s1, t1);
      load_slot(part, g + 2, n_pad, k, teacher, s2, t2);
      load_slot(part, g + 3, n_pad, k, teacher, s3, t3);
      merge3(s0, s1);
      merge3(t0, t1);
      merge3(s2, s3);
      merge3(t2, t3);
      merge3(s0, s2);
      merge3(t0, t2);
      merge3(s, s0);
      merge3(t, t0);
    }
    for (; g < g1; ++g) {
      Stat3 s0, t0;
      load_slot(part, g, n_pad, k, teacher, s0, t0);
      merge3(s, s0);
      merge3(t, t0);
    }
  }
  sh_s[warp][lane] = s;
  sh_t[warp][lane] = t;
  __syncthreads();
  if (warp != 0 || k >= n_live) return;
  for (int w = 1; w < kCombineWarps; ++w) {
    merge3(s, sh_s[w][lane]);
    merge3(t, sh_t[w][lane]);
  }
  const int out = slot_k ? slot_k[k] : k;
  if (out < 0 || !RKL_BOUNDS(out < n_pad)) return;
  const float lse_s = s.m + logf(s.S);
  const float lse_t = teacher ? t.m + logf(t.S) : lse_ext[k];
  const float L = s.A / s.S - lse_s + lse_t;
  saved[3 * out + 0] = lse_s;
  saved[3 * out + 1] = lse_t;
  saved[3 * out + 2] = L;
  if (ent_rows) ent_rows[out] = lse_s - s.Bz / s.S;
  if (lp_rows) lp_rows[out] = tlogit[k] - lse_s;
}

// out[t] = rows[k] if t = row_idx[k] else exactly 0.
__global__ void scatter_rows_kernel(const float* __restrict__ rows, const int32_t* __restrict__ row_idx, int N,
                                    const int32_t* __restrict__ n_dev, long long T, float* __restrict__ out) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  N = live_rows(n_dev, N);
  const int k = lower_bound_i32(row_idx, N, t);
  out[t] = (k < N && row_idx[k] == t) ? rows[k] : 0.f;
}

// loss_tok[t] = L of t if t is trainable else exactly 0.
__global__ void scatter_loss_kernel(const float* __restrict__ saved, const int32_t* __restrict__ row_idx, int N,
                                    const int32_t* __restrict__ n_dev, long long T, float* __restrict__ loss_tok) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  N = live_rows(n_dev, N);
  const int k = lower_bound_i32(row_idx, N, t);
  loss_tok[t] = (k < N && row_idx[k] == t) ? saved[3 * k + 2] : 0.f;
}

__device__ __forceinline__ double block_sum_1024(double v, double* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < 32; ++w) r += sh[w];
  __syncthreads();
  return r;
}

// Scalar loss: token mean sum_k L_k / N, or nested mean over sequences with
// n_b > 0 of sum_{k in b} L_k / n_b.  Fixed summation order (deterministic).
__global__ void __launch_bounds__(1024) reduce_kernel(const float* __restrict__ saved,
                                                      const int32_t* __restrict__ row_idx, int N,
                                                      const int32_t* __restrict__ n_dev, int B, int Sm1,
                                                      int reduction, float* __restrict__ loss) {
  __shared__ double sh[32];
  N = live_rows(n_dev, N);
  if (reduction == 1) {
    double acc = 0.0;
    for (int k = threadIdx.x; k < N; k += 1024) acc += saved[3 * k + 2];
    const double tot = block_sum_1024(acc, sh);
    if (threadIdx.x == 0) *loss = N > 0 ? static_cast<float>(tot / N) : 0.f;
  } else {
    double acc = 0.0, cnt = 0.0;
    for (int b = threadIdx.x; b < B; b += 1024) {
      const int lo = lower_bound_i32(row_idx, N, static_cast<long long>(b) * Sm1);
      const int hi = lower_bound_i32(row_idx, N, static_cast<long long>(b + 1) * Sm1);
      if (hi > lo) {
        double sb = 0.0;
        for (int k = lo; k < hi; ++k) sb += saved[3 * k + 2];
        acc += sb / (hi - lo);
        cnt += 1.0;
      }
    }
    const double tot = block_sum_1024(acc, sh);
    const double c = block_sum_1024(cnt, sh);
    if (threadIdx.x == 0) *loss = c > 0 ? static_cast<float>(tot / c) : 0.f;
  }
}

// --------------------------------------------------------------------- S5
// Row constants of the recompute pass: rowc[0] = lse_s*log2(e),
// rowc[1] = lse_t - lse_s - L, rowc[2] = g = dLoss/dL_k.  Padding rows get 0.
// With a slot map, row p of rowc belongs to compact row slot_k[p].
__global__ void __launch_bounds__(256) row_weights_kernel(const float* __restrict__ saved,
                                                          const int32_t* __restrict__ row_idx, int N,
                                                          const int32_t* __restrict__ n_dev, int n_pad,
                                                          int B, int Sm1, int reduction,
                                                          const float* __restrict__ grad_loss,
                                                          const float* __restrict__ grad_tok,
                                                          float* __restrict__ rowc,
                                                          const int32_t* __restrict__ slot_k) {
  __shared__ int b_eff_sh;
  N = live_rows(n_dev, N);
  if (threadIdx.x == 0) b_eff_sh = 0;
  __syncthreads();
  if (reduction == 2) {
    int local = 0;
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
      const int lo = lower_bound_i32(row_idx, N, static_cast<long long>(b) * Sm1);
      const int hi = lower_bound_i32(row_idx, N, static_cast<long long>(b + 1) * Sm1);
      local += hi > lo;
    }
    atomicAdd(&b_eff_sh, local);
  }
  __syncthreads();
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_pad) return;
  const int k = slot_k ? slot_k[p] : p;
  float c0 = 0.f, c1 = 0.f, c2 = 0.f;
  if (k >= 0 && k < N) {
    const int row = row_idx[k];
    if (!RKL_BOUNDS(row >= 0 && row < B * Sm1)) return;
    const float lse_s = saved[3 * k], lse_t = saved[3 * k + 1], L = saved[3 * k + 2];
    float w = 0.f;
    if (reduction == 1) {
      w = 1.f / static_cast<float>(N);
    } else if (reduction == 2) {
      const int b = row / Sm1;
      const int lo = lower_bound_i32(row_idx, N, static_cast<long long>(b) * Sm1);
      const int hi = lower_bound_i32(row_idx, N, static_cast<long long>(b + 1) * Sm1);
      w = 1.f / (static_cast<float>(b_eff_sh) * static_cast<float>(hi - lo));
    }
    float g = 0.f;
    if (reduction != 0 && grad_loss != nullptr) g = grad_loss[0] * w;
    if (grad_tok != nullptr) g += grad_tok[row];
    c0 = lse_s * kLog2e;
    c1 = lse_t - lse_s - L;
    c2 = g;
  }
  rowc[p] = c0;
  rowc[n_pad + p] = c1;
  rowc[2 * n_pad + p] = c2;
}

// dH_s[t] = dHc[k_slot[k]] (dHc[k] without a slot map) if t = row_idx[k],
// else exact zeros.
__global__ void __launch_bounds__(256) scatter_dh_kernel(const float* __restrict__ dHc,
                                                         const int32_t* __restrict__ row_idx,
                                                         const int32_t* __restrict__ k_slot, int N,
                                                         const int32_t* __restrict__ n_dev, long long T, int H,
                                                         float* __restrict__ dH_s) {
  N = live_rows(n_dev, N);
  for (long long t = blockIdx.x; t < T; t += gridDim.x) {
    const int k = lower_bound_i32(row_idx, N, t);
    const int src = (k < N && row_idx[k] == t) ? (k_slot ? k_slot[k] : k) : -1;
    float* d = dH_s + t * H;
    if (src >= 0) {
      const float* s = dHc + static_cast<long long>(src) * H;
      if ((H & 3) == 0) {
        float4* d4 = reinterpret_cast<float4*>(d);
        const float4* s4 = reinterpret_cast<const float4*>(s);
        for (int i = threadIdx.x; i < H / 4; i += blockDim.x) d4[i] = s4[i];
      } else {
        for (int i = threadIdx.x; i < H; i += blockDim.x) d[i] = s[i];
      }
    } else {
      if ((H & 3) == 0) {
        float4* d4 = reinterpret_cast<float4*>(d);
        for (int i = threadIdx.x; i < H / 4; i += blockDim.x) d4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        for (int i = threadIdx.x; i < H; i += blockDim.x) d[i] = 0.f;
      }
    }
  }
}

// ------------------------------------------------------- teacher per row
// NeMo RL PR #3978, first-version limits: one teacher in the first version,
// with the payload laid out for a per-row teacher index.  Each trainable row
// carries the index of its teacher; rows are regrouped by teacher into whole
// 256-row tiles so that every tile of the tensor-core kernels projects with
// one teacher head.

// counts[g] += trainable rows of teacher g; counts[n] += trainable rows whose
// index is outside [0, n).  Shared-memory histogram, then one global add per
// bin and block (integer adds: the result does not depend on their order).
__global__ void __launch_bounds__(1024) count_teachers_kernel(const uint8_t* __restrict__ mask,
                                                              const int32_t* __restrict__ teacher_idx, long long T,
                                                              int n, int32_t* __restrict__ counts) {
  __shared__ int hist[kMaxTeachers + 1];
  if (threadIdx.x <= kMaxTeachers) hist[threadIdx.x] = 0;
  __syncthreads();
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < T;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (mask[t] != 0) {
      const int g = teacher_idx[t];
      atomicAdd(&hist[(g >= 0 && g < n) ? g : n], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x <= n && hist[threadIdx.x] != 0) atomicAdd(&counts[threadIdx.x], hist[threadIdx.x]);
}

// Teacher-grouped slots.  Compact rows k are taken in ascending order, 1024 at
// a time; a row of teacher g gets slot base[g] + (rows of teacher g before
// it).  Within a warp the rank comes from __match_any_sync, across warps from
// an exclusive scan of the per-warp counts (warp g of the block scans the
// counts of teacher g).  A row whose index is out of range, or whose rank
// exceeds the count given for its teacher, gets no slot (k_slot = -1), so
// every store stays inside the layout even for inconsistent counts.
__global__ void __launch_bounds__(1024) build_slots_kernel(const int32_t* __restrict__ row_idx,
                                                           const int32_t* __restrict__ teacher_idx, int N,
                                                           const TeacherSlots ts, int32_t* __restrict__ slot_k,
                                                           int32_t* __restrict__ k_slot) {
  __shared__ int wcnt[32][kMaxTeachers];  // per warp and teacher; then its exclusive prefix
  __shared__ int total[kMaxTeachers];
  __shared__ int carry[kMaxTeachers];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kMaxTeachers) carry[tid] = 0;
  for (int c0 = 0; c0 < N; c0 += 1024) {
    for (int i = tid; i < 32 * kMaxTeachers; i += 1024) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int k = c0 + tid;
    int g = -1;
    if (k < N) {
      g = teacher_idx[row_idx[k]];
      if (g < 0 || g >= ts.n) g = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, g);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (g >= 0 && rank_w == 0) wcnt[warp][g] = __popc(peers);
    __syncthreads();
    if (warp < ts.n) {
      const int x = wcnt[lane][warp];
      int incl = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      wcnt[lane][warp] = incl - x;
      if (lane == 31) total[warp] = incl;
    }
    __syncthreads();
    if (k < N) {
      int slot = -1;
      if (g >= 0) {
        const int r = carry[g] + wcnt[warp][g] + rank_w;
        if (r < ts.count[g]) {
          slot = ts.base[g] + r;
          slot_k[slot] = k;
        }
      }
      k_slot[k] = slot;
    }
    __syncthreads();
    if (tid < ts.n) carry[tid] += total[tid];
    __syncthreads();
  }
}

// ------------------------------------------------------------ logits pair
// Both sides as [T, V] logits (NeMo RL PR #3978, payload bullet 2: the logits
// path as the numerical reference).  Forward: one CTA per trainable row
// streams z_s and z_t once with 16-byte loads and keeps online
// (m_s, S_s, A, m_t, S_t) per thread, then merges them in a fixed order.
// Backward: one CTA per token row writes dL/dz_s for the whole row (exact
// zeros at masked rows).  Both are pure HBM streams.
struct PairStat {
  float m_s, S_s, A, m_t, S_t;
};

__device__ __forceinline__ void pair_merge(PairStat& a, const PairStat& b) {
  const float ns = fmaxf(a.m_s, b.m_s), nt = fmaxf(a.m_t, b.m_t);
  if (ns != -INFINITY) {
    const float ea = ex2((a.m_s - ns) * kLog2e), eb = ex2((b.m_s - ns) * kLog2e);
    a.S_s = a.S_s * ea + b.S_s * eb;
    a.A = a.A * ea + b.A * eb;
    a.m_s = ns;
  }
  if (nt != -INFINITY) {
    const float ea = ex2((a.m_t - nt) * kLog2e), eb = ex2((b.m_t - nt) * kLog2e);
    a.S_t = a.S_t * ea + b.S_t * eb;
    a.m_t = nt;
  }
}

// Online update with VEC values of each side.
template <int VEC>
__device__ __forceinline__ void pair_update(PairStat& st, const float* xs, const float* xt) {
  float cs = xs[0], ct = xt[0];
#pragma unroll
  for (int j = 1; j < VEC; ++j) {
    cs = fmaxf(cs, xs[j]);
    ct = fmaxf(ct, xt[j]);
  }
  if (cs > st.m_s) {
    const float a = ex2((st.m_s - cs) * kLog2e);
    st.S_s *= a;
    st.A *= a;
    st.m_s = cs;
  }
  if (ct > st.m_t) {
    st.S_t *= ex2((st.m_t - ct) * kLog2e);
    st.m_t = ct;
  }
  const float ms2 = st.m_s * kLog2e, mt2 = st.m_t * kLog2e;
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    const float e = ex2(fmaf(xs[j], kLog2e, -ms2));
    const float f = ex2(fmaf(xt[j], kLog2e, -mt2));
    st.S_s += e;
    st.S_t += f;
    st.A = fmaf(e, xs[j] - xt[j], st.A);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) pair_fwd_kernel(const T* __restrict__ zs_all, const T* __restrict__ zt_all,
                                                       const int32_t* __restrict__ row_idx, int N,
                                                       const int32_t* __restrict__ n_dev, int V,
                                                       float* __restrict__ saved) {
  constexpr int VEC = 16 / sizeof(T);
  const int k = blockIdx.x;
  if (k >= live_rows(n_dev, N)) return;
  const long long r = row_idx[k];
  const T* zs = zs_all + r * V;
  const T* zt = zt_all + r * V;
  PairStat st{-INFINITY, 0.f, 0.f, -INFINITY, 0.f};
  int done = 0;
  if (((reinterpret_cast<uintptr_t>(zs) | reinterpret_cast<uintptr_t>(zt)) & 15) == 0) {
    const int nvec = V / VEC;
    const uint4* vs = reinterpret_cast<const uint4*>(zs);
    const uint4* vt = reinterpret_cast<const uint4*>(zt);
    int i = threadIdx.x;
    for (; i + 256 < nvec; i += 512) {
      const uint4 a0 = ldg_stream_v4(vs + i), b0 = ldg_stream_v4(vt + i);
      const uint4 a1 = ldg_stream_v4(vs + i + 256), b1 = ldg_stream_v4(vt + i + 256);
      float xs[VEC], xt[VEC];
      vec_to_float<T>(a0, xs);
      vec_to_float<T>(b0, xt);
      pair_update<VEC>(st, xs, xt);
      vec_to_float<T>(a1, xs);
      vec_to_float<T>(b1, xt);
      pair_update<VEC>(st, xs, xt);
    }
    for (; i < nvec; i += 256) {
      float xs[VEC], xt[VEC];
      vec_to_float<T>(ldg_stream_v4(vs + i), xs);
      vec_to_float<T>(ldg_stream_v4(vt + i), xt);
      pair_update<VEC>(st, xs, xt);
    }
    done = nvec * VEC;
  }
  for (int v = done + threadIdx.x; v < V; v += 256) {
    const float xs = to_f<T>(zs[v]), xt = to_f<T>(zt[v]);
    pair_update<1>(st, &xs, &xt);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    PairStat b{__shfl_xor_sync(0xffffffffu, st.m_s, o), __shfl_xor_sync(0xffffffffu, st.S_s, o),
               __shfl_xor_sync(0xffffffffu, st.A, o), __shfl_xor_sync(0xffffffffu, st.m_t, o),
               __shfl_xor_sync(0xffffffffu, st.S_t, o)};
    pair_merge(st, b);
  }
  __shared__ PairStat sh[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sh[warp] = st;
  __syncthreads();
  if (threadIdx.x == 0) {
    PairStat t = sh[0];
    for (int w = 1; w < 8; ++w) pair_merge(t, sh[w]);
    const float lse_s = t.m_s + logf(t.S_s);
    const float lse_t = t.m_t + logf(t.S_t);
    saved[3 * k + 0] = lse_s;
    saved[3 * k + 1] = lse_t;
    saved[3 * k + 2] = t.A / t.S_s - lse_s + lse_t;
  }
}

template <typename T>
__device__ __forceinline__ uint4 float_to_vec(const float* d);

template <>
__device__ __forceinline__ uint4 float_to_vec<__nv_bfloat16>(const float* d) {
  return make_uint4(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]), pack_bf16x2(d[4], d[5]),
                    pack_bf16x2(d[6], d[7]));
}

template <>
__device__ __forceinline__ uint4 float_to_vec<float>(const float* d) {
  return make_uint4(__float_as_uint(d[0]), __float_as_uint(d[1]), __float_as_uint(d[2]), __float_as_uint(d[3]));
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// dz[t, :] = g p_s ((z_s - z_t) + lse_t - lse_s - L) for trainable t, else 0.
template <typename T>
__global__ void __launch_bounds__(256) pair_bwd_kernel(const T* __restrict__ zs_all, const T* __restrict__ zt_all,
                                                       const int32_t* __restrict__ row_idx, int N,
                                                       const int32_t* __restrict__ n_dev, int n_pad, int V,
                                                       const float* __restrict__ rowc, T* __restrict__ dz_all) {
  constexpr int VEC = 16 / sizeof(T);
  const long long t = blockIdx.x;
  N = live_rows(n_dev, N);
  const int k = lower_bound_i32(row_idx, N, t);
  const bool hit = k < N && row_idx[k] == t;
  const T* zs = zs_all + t * V;
  const T* zt = zt_all + t * V;
  T* dz = dz_all + t * V;
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(zs) | reinterpret_cast<uintptr_t>(zt) |
                        reinterpret_cast<uintptr_t>(dz)) & 15) == 0;
  const int nvec = vec_ok ? V / VEC : 0;
  if (!hit) {
    uint4* d4 = reinterpret_cast<uint4*>(dz);
    for (int i = threadIdx.x; i < nvec; i += 256) d4[i] = make_uint4(0, 0, 0, 0);
    for (int v = nvec * VEC + threadIdx.x; v < V; v += 256) dz[v] = from_f<T>(0.f);
    return;
  }
  const float lse2 = rowc[k], cst = rowc[n_pad + k], g = rowc[2 * n_pad + k];
  const uint4* vs = reinterpret_cast<const uint4*>(zs);
  const uint4* vt = reinterpret_cast<const uint4*>(zt);
  uint4* vd = reinterpret_cast<uint4*>(dz);
  for (int i = threadIdx.x; i < nvec; i += 256) {
    float xs[VEC], xt[VEC], d[VEC];
    vec_to_float<T>(ldg_stream_v4(vs + i), xs);
    vec_to_float<T>(ldg_stream_v4(vt + i), xt);
#pragma unroll
    for (int j = 0; j < VEC; ++j) d[j] = g * ex2(fmaf(xs[j], kLog2e, -lse2)) * ((xs[j] - xt[j]) + cst);
    vd[i] = float_to_vec<T>(d);
  }
  for (int v = nvec * VEC + threadIdx.x; v < V; v += 256) {
    const float xs = to_f<T>(zs[v]), xt = to_f<T>(zt[v]);
    dz[v] = from_f<T>(g * ex2(fmaf(xs, kLog2e, -lse2)) * ((xs - xt) + cst));
  }
}

}  // namespace

cudaError_t launch_compact(const uint8_t* mask, long long T, int32_t* row_idx, int32_t* n_dev, cudaStream_t s) {
  LaunchScope scope(K_COMPACT, s);
  compact_kernel<<<1, 1024, 0, s>>>(mask, T, row_idx, n_dev);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* h_s, const void* h_t, void* hc_s, void* hc_t, const int32_t* row_idx,
                          const int32_t* slot_k, int n_rows, const int32_t* n_dev, int row_bytes, long long T,
                          cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  LaunchScope scope(K_GATHER, s);
  const int span = n_dev ? ((n_rows + 2 * kBM - 1) / (2 * kBM)) * (2 * kBM) : n_rows;
  dim3 grid(span < 65535 ? span : 65535, h_t ? 2 : 1);
  gather_kernel<<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(h_s), static_cast<const uint8_t*>(h_t),
                                     static_cast<uint8_t*>(hc_s), static_cast<uint8_t*>(hc_t), row_idx, slot_k,
                                     n_rows, n_dev, row_bytes, T);
  return cudaGetLastError();
}

cudaError_t launch_teacher_lse(const void* logits, bool bf16, const int32_t* row_idx, int N, const int32_t* n_dev,
                               int V, long long pitch, float* lse_t, long long rows, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_TEACHER_LSE, s);
  if (bf16)
    teacher_lse_kernel<__nv_bfloat16><<<N, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(logits), row_idx, N, n_dev,
                                                         V, pitch, lse_t, rows);
  else
    teacher_lse_kernel<float><<<N, 256, 0, s>>>(static_cast<const float*>(logits), row_idx, N, n_dev, V, pitch,
                                                lse_t, rows);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* part, int S, int n_pad, int n_rows, const int32_t* n_dev,
                           bool teacher_from_part, const float* lse_ext, const float* tlogit, float* saved,
                           float* ent_rows, float* lp_rows, const int32_t* slot_k, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  LaunchScope scope(K_COMBINE, s);
  combine_kernel<<<(n_rows + 31) / 32, 32 * kCombineWarps, 0, s>>>(part, S, n_pad, n_rows, n_dev,
                                                                   teacher_from_part ? 1 : 0, lse_ext, tlogit,
                                                                   saved, ent_rows, lp_rows, slot_k);
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const float* rows, const int32_t* row_idx, int N, const int32_t* n_dev, long long T,
                                float* out, cudaStream_t s) {
  LaunchScope scope(K_SCATTER_LOSS, s);
  scatter_rows_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, s>>>(rows, row_idx, N, n_dev, T, out);
  return cudaGetLastError();
}

cudaError_t launch_scatter_loss(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, long long T,
                                float* loss_tok, cudaStream_t s) {
  LaunchScope scope(K_SCATTER_LOSS, s);
  scatter_loss_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, s>>>(saved, row_idx, N, n_dev, T, loss_tok);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, int B, int Sm1,
                          int reduction, float* loss, cudaStream_t s) {
  LaunchScope scope(K_REDUCE, s);
  reduce_kernel<<<1, 1024, 0, s>>>(saved, row_idx, N, n_dev, B, Sm1, reduction, loss);
  return cudaGetLastError();
}

cudaError_t launch_row_weights(const float* saved, const int32_t* row_idx, int N, const int32_t* n_dev, int n_pad,
                               int B, int Sm1, int reduction, const float* grad_loss, const float* grad_tok,
                               float* rowc, const int32_t* slot_k, cudaStream_t s) {
  LaunchScope scope(K_ROW_WEIGHTS, s);
  row_weights_kernel<<<(n_pad + 255) / 256, 256, 0, s>>>(saved, row_idx, N, n_dev, n_pad, B, Sm1, reduction,
                                                         grad_loss, grad_tok, rowc, slot_k);
  return cudaGetLastError();
}

cudaError_t launch_scatter_dh(const float* dHc, const int32_t* row_idx, const int32_t* k_slot, int N,
                              const int32_t* n_dev, long long T, int H, float* dH_s, cudaStream_t s) {
  LaunchScope scope(K_SCATTER_DH, s);
  const long long blocks = T < 65535 * 8 ? T : 65535 * 8;
  scatter_dh_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(dHc, row_idx, k_slot, N, n_dev, T, H, dH_s);
  return cudaGetLastError();
}

cudaError_t launch_count_teachers(const uint8_t* mask, const int32_t* teacher_idx, long long T, int n_teachers,
                                  int32_t* counts, cudaStream_t s) {
  LaunchScope scope(K_COUNT_TEACHERS, s);
  const long long blocks = (T + 1023) / 1024;
  count_teachers_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 1024, 0, s>>>(mask, teacher_idx, T,
                                                                                               n_teachers, counts);
  return cudaGetLastError();
}

cudaError_t launch_build_slots(const int32_t* row_idx, const int32_t* teacher_idx, int N, const TeacherSlots& ts,
                               int32_t* slot_k, int32_t* k_slot, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_BUILD_SLOTS, s);
  build_slots_kernel<<<1, 1024, 0, s>>>(row_idx, teacher_idx, N, ts, slot_k, k_slot);
  return cudaGetLastError();
}

}  // namespace rkl

namespace rkl {

cudaError_t launch_pair_fwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx, int N,
                            const int32_t* n_dev, int V, float* saved, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  LaunchScope scope(K_PAIR_FWD, s);
  if (bf16)
    pair_fwd_kernel<__nv_bfloat16><<<N, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(zs),
                                                      static_cast<const __nv_bfloat16*>(zt), row_idx, N, n_dev, V,
                                                      saved);
  else
    pair_fwd_kernel<float><<<N, 256, 0, s>>>(static_cast<const float*>(zs), static_cast<const float*>(zt), row_idx,
                                             N, n_dev, V, saved);
  return cudaGetLastError();
}

cudaError_t launch_pair_bwd(const void* zs, const void* zt, bool bf16, const int32_t* row_idx, int N,
                            const int32_t* n_dev, int n_pad, long long T, int V, const float* rowc, void* dz,
                            cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  LaunchScope scope(K_PAIR_BWD, s);
  if (bf16)
    pair_bwd_kernel<__nv_bfloat16><<<static_cast<unsigned>(T), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(zs), static_cast<const __nv_bfloat16*>(zt), row_idx, N, n_dev, n_pad, V,
        rowc, static_cast<__nv_bfloat16*>(dz));
  else
    pair_bwd_kernel<float><<<static_cast<unsigned>(T), 256, 0, s>>>(static_cast<const float*>(zs),
                                                                    static_cast<const float*>(zt), row_idx, N, n_dev,
                                                                    n_pad, V, rowc, static_cast<float*>(dz));
  return cudaGetLastError();
}

}  // namespace rkl
