// api.cu -- the C ABI of librkl.so (declared in include/rkl.h).
//
// Argument validation, workspace layout, TMA descriptor encoding, per-device
// one-time setup and the launch sequence of each entry point.  Every numeric
// step runs in the kernels of tc_kernels.cu / small_kernels.cu /
// simt_kernels.cu; nothing here touches tensor data on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "rkl.h"
#include "kernels.h"

namespace rkl {

// An NVTX range over one C-ABI call, named after the entry point.  Profilers
// that listen to NVTX (Nsight Systems, Nsight Compute's range filters) show
// each call with its kernels under it; without one attached a push/pop costs
// a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define RKL_NVTX_RANGE() ::rkl::NvtxRange rkl_nvtx_range_(__func__)

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error;

static rkl_status fail(rkl_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define RKL_CUDA(call)                                                                          \
  do {                                                                                          \
    cudaError_t e__ = (call);                                                                   \
    if (e__ != cudaSuccess) return fail(RKL_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e__)); \
  } while (0)

// ------------------------------------------------------------------ profiling
static const char* const kKernelNames[K_COUNT] = {
    "compact_rows", "gather_rows",   "fwd_dual_tc",  "fwd_single_tc", "teacher_lse", "combine_splits",
    "scatter_loss", "reduce_loss",   "row_weights",  "dz_dual_tc",    "dz_single_tc", "grad_dw_dh_tc",
    "scatter_dh",   "fwd_simt_fp32", "dz_simt_fp32", "grad_simt_fp32", "pair_fwd",   "pair_bwd",
    "count_teachers", "build_slots", "topk_fwd", "topk_bwd", "zw_dual_tc", "dz_topk_tc", "topk_rowk",
    "zw_single_tc", "dz_topk_single_tc"};

const char* kernel_name(int id) { return (id >= 0 && id < K_COUNT) ? kKernelNames[id] : nullptr; }

struct ProfRec {
  int id;
  cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static std::atomic<bool> g_profile{false};
static std::atomic<long long> g_launches{0};
static std::vector<ProfRec> g_prof_pending;
static double g_prof_ms[K_COUNT];
static long long g_prof_n[K_COUNT];

LaunchScope::LaunchScope(int id_, cudaStream_t s) : id(id_), stream(s) {
  g_launches.fetch_add(1);
  if (g_profile.load()) {
    if (cudaEventCreate(&ev0) == cudaSuccess && cudaEventCreate(&ev1) == cudaSuccess) {
      cudaEventRecord(ev0, s);
    } else {
      ev0 = ev1 = nullptr;
    }
  }
}

LaunchScope::~LaunchScope() {
  if (ev0 && ev1) {
    cudaEventRecord(ev1, stream);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_pending.push_back({id, ev0, ev1});
  }
}

// ------------------------------------------------------------------ devices
struct DevState {
  bool ready = false;
  int sms = 0;
};
static std::mutex g_dev_mu;
static DevState g_devs[64];

static rkl_status device_setup(int* sms) {
  int dev = 0;
  RKL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RKL_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState& d = g_devs[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    RKL_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    RKL_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (major != 10 || minor != 0)
      return fail(RKL_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev, major,
                  minor);
    RKL_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    RKL_CUDA(tc_setup(dev));
    d.ready = true;
  }
  *sms = d.sms;
  return RKL_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major map: `inner` contiguous elements per row, `outer` rows,
// `pitch` bytes between rows; 128-byte swizzle; out-of-bounds reads give 0.
static rkl_status make_map(CUtensorMap* m, const void* ptr, bool f32, uint64_t inner, uint64_t outer,
                           uint64_t pitch, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(RKL_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(RKL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %llux%llu pitch %llu box %ux%u", (int)r,
                (unsigned long long)inner, (unsigned long long)outer, (unsigned long long)pitch, box_inner,
                box_outer);
  return RKL_OK;
}

// ------------------------------------------------------------------ plan
constexpr int kVcBf16 = 65536;  // widest vocab chunk of the backward (multiple of kFBN)
constexpr int kVcF32 = 1024;
constexpr int kSimtSplits = 37;

struct Plan {
  int n_pad = 0, es = 2, S = 1, VT = 1, Vc = 0, nchunks = 1;
  size_t off_hcs = 0, off_hct = 0, off_part = 0, off_rowc = 0, off_lse = 0, off_dz = 0, off_dh = 0, off_cnt = 0,
         off_slot = 0, off_kslot = 0, off_rowk = 0, off_z = 0, total = 0;
  int zrows = 0;      // top-k, hidden payload: rows of a logit block
  long long zpitch = 0;  // its row pitch (floats)
};

constexpr int kTopkBlockRows = 2048;  // top-k, hidden payload: rows whose logits are written at a time

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout.  S = number of partial-statistics groups of the forward:
// groups of kGroupTiles vocab tiles on the tensor-core path, kSimtSplits
// vocab splits on the fp32 path -- both depend on V only.  With a teacher per
// row (n_teachers > 1) the rows are regrouped by teacher into whole 256-row
// tiles: sum_g ceil(n_g / 256) <= ceil(N / 256) + n_teachers - 1 tiles, plus
// the slot maps.
static Plan make_plan(rkl_payload payload, rkl_dtype dtype, int64_t n_max, int64_t H, int64_t V,
                      int n_teachers = 1) {
  Plan p;
  const bool bf16 = dtype == RKL_BF16;
  const int tile_v = bf16 ? kFBN : kSimtBN;
  p.es = bf16 ? 2 : 4;
  const int64_t n = n_max < 1 ? 1 : n_max;
  p.n_pad = static_cast<int>(((n + 2 * kBM - 1) / (2 * kBM)) * (2 * kBM));  // whole 256-row pair tiles
  if (n_teachers > 1) p.n_pad += 2 * kBM * (n_teachers - 1);
  p.VT = static_cast<int>((V + tile_v - 1) / tile_v);
  // tensor-core path: fwd_slots statistics slots (column parts) per group of
  // the forward kernel of this payload (two GEMMs on the hidden payloads)
  const int ng = (payload == RKL_PAYLOAD_HIDDEN || payload == RKL_PAYLOAD_TOPK_HIDDEN) ? 2 : 1;
  p.S = bf16 ? fwd_slots(ng) * ((p.VT + kGroupTiles - 1) / kGroupTiles) : (p.VT < kSimtSplits ? p.VT : kSimtSplits);
  // Backward vocab chunks: as few as the widest chunk allows, of equal width
  // (a multiple of the 256-column tile), so that every gradient launch has the
  // same work and the tails of the persistent kernels are paid few times.
  const int vc = bf16 ? kVcBf16 : kVcF32;
  const int64_t vround = ((V + kFBN - 1) / kFBN) * kFBN;
  if (bf16) {
    const int64_t nch = (vround + vc - 1) / vc;
    const int64_t w = (vround + nch - 1) / nch;
    p.Vc = static_cast<int>(((w + kFBN - 1) / kFBN) * kFBN);
  } else {
    p.Vc = static_cast<int>(vround < vc ? vround : vc);
  }
  p.nchunks = static_cast<int>((V + p.Vc - 1) / p.Vc);
  size_t off = 256;  // header
  p.off_hcs = off;
  off = align256(off + size_t(p.n_pad) * H * p.es);
  p.off_hct = off;
  if (payload == RKL_PAYLOAD_HIDDEN || payload == RKL_PAYLOAD_TOPK_HIDDEN)
    off = align256(off + size_t(p.n_pad) * H * p.es);
  p.off_part = off;
  off = align256(off + size_t(p.S) * kStatVals * p.n_pad * sizeof(float));
  p.off_rowc = off;
  off = align256(off + size_t(3) * p.n_pad * sizeof(float));
  p.off_lse = off;
  off = align256(off + size_t(p.n_pad) * sizeof(float));
  p.off_dz = off;
  off = align256(off + size_t(p.n_pad) * p.Vc * p.es);
  p.off_dh = off;
  off = align256(off + size_t(p.n_pad) * H * sizeof(float));
  p.off_cnt = off;
  off = align256(off + size_t(p.nchunks) * sizeof(int));
  if (n_teachers > 1) {
    p.off_slot = off;
    off = align256(off + size_t(p.n_pad) * sizeof(int32_t));
    p.off_kslot = off;
    off = align256(off + size_t(n) * sizeof(int32_t));
  }
  if (payload == RKL_PAYLOAD_TOPK_HIDDEN || payload == RKL_PAYLOAD_TOPK_LOGITS) {
    // per-row constants of the top-k dz pass, and the fp32 z_s (hidden
    // payload: and z_t) of one block of rows: never more than
    // kTopkBlockRows rows of logits at a time.  The teacher-logits payload
    // selects against the shipped bf16 teacher rows directly.
    p.off_rowk = off;
    off = align256(off + size_t(6) * p.n_pad * sizeof(float));
    p.zrows = p.n_pad < kTopkBlockRows ? p.n_pad : kTopkBlockRows;
    p.zpitch = ((V + 3) / 4) * 4;
    p.off_z = off;
    const size_t zblocks = payload == RKL_PAYLOAD_TOPK_HIDDEN ? 2 : 1;
    off = align256(off + zblocks * p.zrows * p.zpitch * sizeof(float));
  }
  p.total = off;
  return p;
}

// Teacher-grouped row layout of the per-row-teacher mode (host side).
struct MultiTeacher {
  int n = 0;                         // teachers (> 1)
  const int32_t* teacher_idx = nullptr;  // [B, Sm1] device
  const void* W_t = nullptr;         // stacked heads [n, V, H]
  TeacherSlots ts{};
  int n_rows = 0;                    // slots in use (sum of 256-rounded counts)
  int group_row_end[kMaxTeachers] = {};
};

static rkl_status make_multi(int n_teachers, const int32_t* teacher_idx, const int32_t* counts, int32_t N,
                             MultiTeacher* mt) {
  if (n_teachers < 1 || n_teachers > kMaxTeachers)
    return fail(RKL_ERR_SHAPE, "n_teachers = %d outside [1, %d]", n_teachers, kMaxTeachers);
  if (teacher_idx == nullptr || counts == nullptr) return fail(RKL_ERR_NULL, "teacher_idx and counts must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(teacher_idx) & 15) != 0)
    return fail(RKL_ERR_ALIGN, "teacher_idx is not 16-byte aligned");
  mt->n = n_teachers;
  mt->teacher_idx = teacher_idx;
  mt->ts.n = n_teachers;
  long long sum = 0;
  int base = 0;
  for (int g = 0; g < n_teachers; ++g) {
    if (counts[g] < 0) return fail(RKL_ERR_SHAPE, "counts[%d] = %d is negative", g, counts[g]);
    sum += counts[g];
    mt->ts.count[g] = counts[g];
    mt->ts.base[g] = base;
    if (sum > N) break;
    base += ((counts[g] + 2 * kBM - 1) / (2 * kBM)) * (2 * kBM);
    mt->group_row_end[g] = base;
  }
  if (sum != N)
    return fail(RKL_ERR_SHAPE,
                "per-teacher counts add up to %lld but N = %d (a trainable row has a teacher index outside "
                "[0, n_teachers), or the counts belong to another mask)",
                sum, N);
  mt->n_rows = base;
  return RKL_OK;
}

// ------------------------------------------------------------------ checks
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static rkl_status check_common(rkl_payload payload, rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                               int32_t N, int reduction) {
  if (dtype != RKL_BF16 && dtype != RKL_FP32) return fail(RKL_ERR_DTYPE, "unknown dtype %d", (int)dtype);
  if (payload != RKL_PAYLOAD_HIDDEN && payload != RKL_PAYLOAD_LOGITS && payload != RKL_PAYLOAD_LOGITS_PAIR &&
      payload != RKL_PAYLOAD_TOPK_HIDDEN && payload != RKL_PAYLOAD_TOPK_LOGITS)
    return fail(RKL_ERR_DTYPE, "unknown payload %d", (int)payload);
  if (payload == RKL_PAYLOAD_LOGITS_PAIR) H = 64;  // no hidden dimension in this mode
  if (reduction < 0 || reduction > 2) return fail(RKL_ERR_DTYPE, "unknown reduction %d", reduction);
  if (B < 1 || Sm1 < 1 || H < 1 || V < 1) return fail(RKL_ERR_SHAPE, "B, Sm1, H, V must be >= 1");
  if (B * Sm1 >= (int64_t(1) << 31)) return fail(RKL_ERR_SHAPE, "B*Sm1 = %lld exceeds 2^31-1", (long long)(B * Sm1));
  if (H > 65536) return fail(RKL_ERR_SHAPE, "H = %lld exceeds 65536", (long long)H);
  if (V >= (int64_t(1) << 30)) return fail(RKL_ERR_SHAPE, "V = %lld too large", (long long)V);
  if (N < 0 || N > B * Sm1) return fail(RKL_ERR_SHAPE, "N = %d outside [0, B*Sm1]", N);
  if (dtype == RKL_BF16) {
    if (H % 64 != 0) return fail(RKL_ERR_SHAPE, "bf16 requires H %% 64 == 0 (H = %lld)", (long long)H);
    if ((payload == RKL_PAYLOAD_LOGITS || payload == RKL_PAYLOAD_TOPK_LOGITS) && V % 8 != 0)
      return fail(RKL_ERR_SHAPE, "bf16 logits payload requires V %% 8 == 0 (V = %lld)", (long long)V);
  }
  return RKL_OK;
}

static rkl_status check_ptr(const void* p, const char* name, bool required = true) {
  if (p == nullptr) return required ? fail(RKL_ERR_NULL, "%s is NULL", name) : RKL_OK;
  if (!aligned16(p)) return fail(RKL_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return RKL_OK;
}

// The optional device row count: one int32, 4-byte aligned.
static rkl_status check_n_dev(const int32_t* n_dev) {
  if (n_dev != nullptr && (reinterpret_cast<uintptr_t>(n_dev) & 3) != 0)
    return fail(RKL_ERR_ALIGN, "n_dev is not 4-byte aligned");
  return RKL_OK;
}

#define RKL_TRY(x)                   \
  do {                               \
    rkl_status s__ = (x);            \
    if (s__ != RKL_OK) return s__;   \
  } while (0)

static uint8_t* ws_at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// ------------------------------------------------------------------ forward
static rkl_status forward_impl(rkl_payload payload, const void* h_s, const void* teacher, const void* W_s,
                               const void* W_t, rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                               const int32_t* row_idx, int32_t N, const int32_t* n_dev, rkl_reduction reduction,
                               float* loss_tok, float* loss, float* saved, void* workspace, size_t workspace_bytes,
                               void* stream_, bool forward_only_workspace = false, const int32_t* targets = nullptr,
                               float* entropy = nullptr, float* target_logprob = nullptr,
                               const MultiTeacher* mt = nullptr) {
  RKL_TRY(check_common(payload, dtype, B, Sm1, H, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  if (mt && n_dev)
    return fail(RKL_ERR_UNSUPPORTED, "a teacher per row needs the per-teacher counts on the host (n_dev must be NULL)");
  RKL_TRY(check_ptr(h_s, "h_s"));
  RKL_TRY(check_ptr(teacher, payload == RKL_PAYLOAD_HIDDEN ? "h_t" : "teacher_logits"));
  RKL_TRY(check_ptr(W_s, "W_s"));
  if (payload == RKL_PAYLOAD_HIDDEN) RKL_TRY(check_ptr(W_t, "W_t"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(loss_tok, "loss_tok", false));
  RKL_TRY(check_ptr(loss, "loss", false));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(workspace, "workspace"));
  RKL_TRY(check_ptr(targets, "targets", false));
  RKL_TRY(check_ptr(entropy, "entropy", false));
  RKL_TRY(check_ptr(target_logprob, "target_logprob", false));
  if (target_logprob && !targets) return fail(RKL_ERR_NULL, "target_logprob needs targets");
  const Plan pl = make_plan(payload, dtype, N, H, V, mt ? mt->n : 1);
  // The forward touches only the regions in front of the dz chunk.
  const size_t needed = forward_only_workspace ? pl.off_dz : pl.total;
  if (workspace_bytes < needed)
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, needed);
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  const long long T = B * Sm1;
  const bool bf16 = dtype == RKL_BF16;
  const bool hidden = payload == RKL_PAYLOAD_HIDDEN;

  // Per-row entropy / target log-prob reuse regions of the backward's row
  // constants (3 x n_pad floats), which the forward does not otherwise use.
  float* rowc = reinterpret_cast<float*>(ws_at(workspace, pl.off_rowc));
  float* tlogit = targets ? rowc : nullptr;
  float* ent_rows = entropy ? rowc + pl.n_pad : nullptr;
  float* lp_rows = target_logprob ? rowc + 2 * pl.n_pad : nullptr;
  // A target id outside [0, V) is never found by the kernels: its log-prob
  // reads back the NaN written here.
  if (tlogit && N > 0) RKL_CUDA(cudaMemsetAsync(tlogit, 0xFF, size_t(pl.n_pad) * sizeof(float), s));
  if (N > 0) {
    float* part = reinterpret_cast<float*>(ws_at(workspace, pl.off_part));
    float* lse_ext = reinterpret_cast<float*>(ws_at(workspace, pl.off_lse));
    // Teacher per row: rows regrouped by teacher into whole pair tiles.
    int32_t* slot_k = nullptr;
    int n_rows = N;
    if (mt) {
      slot_k = reinterpret_cast<int32_t*>(ws_at(workspace, pl.off_slot));
      n_rows = mt->n_rows;
      RKL_CUDA(cudaMemsetAsync(slot_k, 0xFF, size_t(n_rows) * sizeof(int32_t), s));
      RKL_CUDA(launch_build_slots(row_idx, mt->teacher_idx, N, mt->ts, slot_k,
                                  reinterpret_cast<int32_t*>(ws_at(workspace, pl.off_kslot)), s));
    }
    // S2: compact the rows (skipped when every row is known to be trainable).
    const bool identity = N == T && !mt && !n_dev;
    const void* as = h_s;
    const void* at = teacher;
    if (!identity) {
      as = ws_at(workspace, pl.off_hcs);
      at = hidden ? ws_at(workspace, pl.off_hct) : nullptr;
      RKL_CUDA(launch_gather(h_s, hidden ? teacher : nullptr, const_cast<void*>(as), const_cast<void*>(at), row_idx,
                             slot_k, n_rows, n_dev, static_cast<int>(H * pl.es), T, s));
    }
    // S8: teacher log-sum-exp from the shipped logits.
    if (!hidden)
      RKL_CUDA(launch_teacher_lse(teacher, bf16, row_idx, N, n_dev, static_cast<int>(V), V, lse_ext, T, s));
    const int ng = hidden ? 2 : 1;
    if (bf16) {
      FusedArgs a;
      memset(&a, 0, sizeof(a));
      RKL_TRY(make_map(&a.tm_as, as, false, H, n_rows, H * 2, kBK, kBM));
      RKL_TRY(make_map(&a.tm_bs, W_s, false, H, V, H * 2, kBK, kFBN / 2));
      if (hidden) {
        RKL_TRY(make_map(&a.tm_at, at, false, H, n_rows, H * 2, kBK, kBM));
        RKL_TRY(make_map(&a.tm_bt, W_t, false, H, V * (mt ? mt->n : 1), H * 2, kBK, kFBN / 2));
        if (mt) {
          a.tgroups = mt->n;
          for (int g = 0; g < mt->n; ++g) a.group_row_end[g] = mt->group_row_end[g];
        }
      } else {
        a.teacher = static_cast<const uint16_t*>(teacher);
        a.teacher_rows = identity ? nullptr : row_idx;
        a.teacher_pitch = V;
      }
      a.part = part;
      a.row_idx = row_idx;
      a.targets = targets;
      a.tlogit = tlogit;
      a.N = n_rows;
      a.n_dev = n_dev;
      a.n_pad = pl.n_pad;
      a.H = static_cast<int>(H);
      a.V = static_cast<int>(V);
      a.KB = static_cast<int>(H / kBK);
      a.IT = pl.VT;
      a.vt_base = 0;
      a.GT = kGroupTiles;
      a.G = pl.S / fwd_slots(ng);
      const int units = ((n_rows + 2 * kBM - 1) / (2 * kBM)) * a.G;  // at most; the kernel takes the live count
      RKL_CUDA(launch_fused(ng, false, a, 2 * units < sms ? 2 * units : sms, s));
    } else {
      SimtArgs a;
      memset(&a, 0, sizeof(a));
      a.as = static_cast<const float*>(as);
      a.bs = static_cast<const float*>(W_s);
      if (hidden) {
        a.at = static_cast<const float*>(at);
        a.bt = static_cast<const float*>(W_t);
        if (mt) {
          a.tgroups = mt->n;
          for (int g = 0; g < mt->n; ++g) a.group_row_end[g] = mt->group_row_end[g];
        }
      } else {
        a.teacher = static_cast<const float*>(teacher);
        a.teacher_rows = identity ? nullptr : row_idx;
        a.teacher_pitch = V;
      }
      a.part = part;
      a.row_idx = row_idx;
      a.targets = targets;
      a.tlogit = tlogit;
      a.N = n_rows;
      a.n_dev = n_dev;
      a.n_pad = pl.n_pad;
      a.H = static_cast<int>(H);
      a.V = static_cast<int>(V);
      a.IT = pl.VT;
      a.S = pl.S;
      a.ng = ng;
      const int MT = (n_rows + kSimtBN - 1) / kSimtBN;
      RKL_CUDA(launch_simt_fused(false, a, dim3(MT, pl.S), s));
    }
    // S4
    RKL_CUDA(launch_combine(part, pl.S, pl.n_pad, n_rows, n_dev, hidden, lse_ext, tlogit, saved, ent_rows, lp_rows,
                            slot_k, s));
  }
  if (loss_tok) RKL_CUDA(launch_scatter_loss(saved, row_idx, N, n_dev, T, loss_tok, s));
  if (entropy) RKL_CUDA(launch_scatter_rows(ent_rows, row_idx, N, n_dev, T, entropy, s));
  if (target_logprob) RKL_CUDA(launch_scatter_rows(lp_rows, row_idx, N, n_dev, T, target_logprob, s));
  if (loss && reduction != RKL_REDUCE_NONE)
    RKL_CUDA(launch_reduce(saved, row_idx, N, n_dev, static_cast<int>(B), static_cast<int>(Sm1), reduction, loss, s));
  return RKL_OK;
}

// ------------------------------------------------------------------ backward
static rkl_status backward_impl(rkl_payload payload, const void* h_s, const void* teacher, const void* W_s,
                                const void* W_t, rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                const int32_t* row_idx, int32_t N, const int32_t* n_dev, rkl_reduction reduction,
                                const float* saved, const float* grad_loss, const float* grad_tok, float* dH_s,
                                float* dW_s, void* workspace, size_t workspace_bytes, void* stream_,
                                const MultiTeacher* mt = nullptr, const int32_t* topk_targets = nullptr) {
  RKL_TRY(check_common(payload, dtype, B, Sm1, H, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  if (mt && n_dev)
    return fail(RKL_ERR_UNSUPPORTED, "a teacher per row needs the per-teacher counts on the host (n_dev must be NULL)");
  const bool topk = payload == RKL_PAYLOAD_TOPK_HIDDEN || payload == RKL_PAYLOAD_TOPK_LOGITS;
  const bool hidden = payload == RKL_PAYLOAD_HIDDEN || payload == RKL_PAYLOAD_TOPK_HIDDEN;
  RKL_TRY(check_ptr(h_s, "h_s"));
  RKL_TRY(check_ptr(teacher, hidden ? "h_t" : "teacher_logits"));
  RKL_TRY(check_ptr(W_s, "W_s"));
  if (hidden) RKL_TRY(check_ptr(W_t, "W_t"));
  if (topk && dtype != RKL_BF16)
    return fail(RKL_ERR_UNSUPPORTED, "the top-k estimator on the tensor-core payloads needs bf16 inputs");
  if (topk) RKL_TRY(check_ptr(topk_targets, "targets"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(grad_loss, "grad_loss", false));
  RKL_TRY(check_ptr(grad_tok, "grad_tok", false));
  RKL_TRY(check_ptr(dH_s, "dH_s"));
  RKL_TRY(check_ptr(dW_s, "dW_s"));
  RKL_TRY(check_ptr(workspace, "workspace"));
  const Plan pl = make_plan(payload, dtype, N, H, V, mt ? mt->n : 1);
  if (workspace_bytes < pl.total)
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, pl.total);
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  const long long T = B * Sm1;
  const bool bf16 = dtype == RKL_BF16;
  float* dHc = reinterpret_cast<float*>(ws_at(workspace, pl.off_dh));

  if (N == 0) {
    RKL_CUDA(cudaMemsetAsync(dW_s, 0, size_t(V) * H * sizeof(float), s));
    RKL_CUDA(launch_scatter_dh(dHc, row_idx, nullptr, 0, nullptr, T, static_cast<int>(H), dH_s, s));
    return RKL_OK;
  }
  // Teacher per row: rows regrouped by teacher into whole pair tiles.
  int32_t* slot_k = nullptr;
  int32_t* k_slot = nullptr;
  int n_rows = N;
  if (mt) {
    slot_k = reinterpret_cast<int32_t*>(ws_at(workspace, pl.off_slot));
    k_slot = reinterpret_cast<int32_t*>(ws_at(workspace, pl.off_kslot));
    n_rows = mt->n_rows;
    RKL_CUDA(cudaMemsetAsync(slot_k, 0xFF, size_t(n_rows) * sizeof(int32_t), s));
    RKL_CUDA(launch_build_slots(row_idx, mt->teacher_idx, N, mt->ts, slot_k, k_slot, s));
  }
  const bool identity = N == T && !mt && !n_dev;
  const void* as = h_s;
  const void* at = teacher;
  if (!identity) {
    as = ws_at(workspace, pl.off_hcs);
    at = hidden ? ws_at(workspace, pl.off_hct) : nullptr;
    RKL_CUDA(launch_gather(h_s, hidden ? teacher : nullptr, const_cast<void*>(as), const_cast<void*>(at), row_idx,
                           slot_k, n_rows, n_dev, static_cast<int>(H * pl.es), T, s));
  }
  float* rowc = reinterpret_cast<float*>(ws_at(workspace, pl.off_rowc));
  RKL_CUDA(launch_row_weights(saved, row_idx, N, n_dev, pl.n_pad, static_cast<int>(B), static_cast<int>(Sm1),
                              reduction, grad_loss, grad_tok, rowc, slot_k, s));
  float* rowk = nullptr;
  if (topk) {
    rowk = reinterpret_cast<float*>(ws_at(workspace, pl.off_rowk));
    RKL_CUDA(launch_topk_rowk(saved, saved + 3 * size_t(N), row_idx, topk_targets, N, n_dev, pl.n_pad, rowk, s));
  }
  void* dz = ws_at(workspace, pl.off_dz);
  const int ng = hidden ? 2 : 1;
  const int nchunks = static_cast<int>((V + pl.Vc - 1) / pl.Vc);

  if (bf16) {
    FusedArgs a;
    memset(&a, 0, sizeof(a));
    RKL_TRY(make_map(&a.tm_as, as, false, H, n_rows, H * 2, kBK, kBM));
    RKL_TRY(make_map(&a.tm_bs, W_s, false, H, V, H * 2, kBK, kFBN / 2));
    if (hidden) {
      RKL_TRY(make_map(&a.tm_at, at, false, H, n_rows, H * 2, kBK, kBM));
      RKL_TRY(make_map(&a.tm_bt, W_t, false, H, V * (mt ? mt->n : 1), H * 2, kBK, kFBN / 2));
      if (mt) {
        a.tgroups = mt->n;
        for (int g = 0; g < mt->n; ++g) a.group_row_end[g] = mt->group_row_end[g];
      }
    } else {
      a.teacher = static_cast<const uint16_t*>(teacher);
      a.teacher_rows = identity ? nullptr : row_idx;
      a.teacher_pitch = V;
    }
    a.rowc = rowc;
    a.rowk = rowk;
    a.N = n_rows;
    a.n_dev = n_dev;
    a.n_pad = pl.n_pad;
    a.H = static_cast<int>(H);
    a.V = static_cast<int>(V);
    a.KB = static_cast<int>(H / kBK);
    const int MT = (n_rows + 2 * kBM - 1) / (2 * kBM);  // at most; the kernels take the live count

    int* counters = reinterpret_cast<int*>(ws_at(workspace, pl.off_cnt));
    RKL_CUDA(cudaMemsetAsync(counters, 0, size_t(nchunks) * sizeof(int), s));
    GradArgs g;
    memset(&g, 0, sizeof(g));
    RKL_TRY(make_map(&g.tm_hs_mn, as, false, H, n_rows, H * 2, 64, 64));
    RKL_TRY(make_map(&g.tm_ws_mn, W_s, false, H, V, H * 2, 64, 64));
    RKL_TRY(make_map(&g.tm_dw, dW_s, true, H, V, H * 4, 32, 32));
    RKL_TRY(make_map(&g.tm_dh, dHc, true, H, n_rows, H * 4, 32, 32));
    g.N = n_rows;
    g.n_dev = n_dev;
    g.dw = dW_s;
    g.dh = dHc;
    g.dw_rows = static_cast<int>(V);
    g.dh_rows = n_rows;
    g.H = static_cast<int>(H);
    g.NT = static_cast<int>(H / kGradBN) + (H % kGradBN ? 1 : 0);

    for (int c = 0; c < nchunks; ++c) {
      const int cv0 = c * pl.Vc;
      const int cw = static_cast<int>((V - cv0) < pl.Vc ? (V - cv0) : pl.Vc);
      // S6: recompute the logits of this chunk and write dz (bf16) [N, cw].
      RKL_TRY(make_map(&a.tm_dz, dz, false, cw, n_rows, size_t(pl.Vc) * 2, 64, 32));
      a.IT = (cw + kFBN - 1) / kFBN;
      a.vt_base = cv0 / kFBN;
      a.chunk_v0 = cv0;
      a.GT = 1;
      a.G = a.IT;
      const int units = MT * a.IT;
      const int fgrid = 2 * units < sms ? 2 * units : sms;
      if (topk)
        RKL_CUDA(launch_fused_topk(2, ng, a, fgrid, s));
      else
        RKL_CUDA(launch_fused(ng, true, a, fgrid, s));
      // S7: dW_s[chunk] = dz^T hc_s and dHc (+)= dz W_s[chunk].
      RKL_TRY(make_map(&g.tm_dz_k, dz, false, cw, n_rows, size_t(pl.Vc) * 2, 64, 128));
      RKL_TRY(make_map(&g.tm_dz_mn, dz, false, cw, n_rows, size_t(pl.Vc) * 2, 64, 64));
      g.cw = cw;
      g.cv0 = cv0;
      g.MTW = (cw + 2 * kBM - 1) / (2 * kBM);
      g.nW = g.MTW * g.NT;
      g.KBH = (cw + kBK - 1) / kBK;
      g.dh_accumulate = c > 0;
      g.tile_counter = counters + c;
      const int pairs = g.nW + MT * g.NT;  // at most
      RKL_CUDA(launch_grad(g, 2 * pairs < sms ? 2 * pairs : sms, s));
    }
  } else {
    SimtArgs a;
    memset(&a, 0, sizeof(a));
    a.as = static_cast<const float*>(as);
    a.bs = static_cast<const float*>(W_s);
    if (hidden) {
      a.at = static_cast<const float*>(at);
      a.bt = static_cast<const float*>(W_t);
      if (mt) {
        a.tgroups = mt->n;
        for (int g = 0; g < mt->n; ++g) a.group_row_end[g] = mt->group_row_end[g];
      }
    } else {
      a.teacher = static_cast<const float*>(teacher);
      a.teacher_rows = identity ? nullptr : row_idx;
      a.teacher_pitch = V;
    }
    a.rowc = rowc;
    a.dz = static_cast<float*>(dz);
    a.N = n_rows;
    a.n_dev = n_dev;
    a.n_pad = pl.n_pad;
    a.H = static_cast<int>(H);
    a.V = static_cast<int>(V);
    a.ng = ng;
    const int MT = (n_rows + kSimtBN - 1) / kSimtBN;
    for (int c = 0; c < nchunks; ++c) {
      const int cv0 = c * pl.Vc;
      const int cw = static_cast<int>((V - cv0) < pl.Vc ? (V - cv0) : pl.Vc);
      a.cw = cw;
      a.IT = (cw + kSimtBN - 1) / kSimtBN;
      a.vt_base = cv0 / kSimtBN;
      a.chunk_v0 = cv0;
      const int items = MT * a.IT;
      RKL_CUDA(launch_simt_fused(true, a, dim3(items < 4 * sms ? items : 4 * sms), s));
      const float* dzf = static_cast<const float*>(dz);
      // dW_s[cv0 + m, n] = sum_k dz[k, m] hc_s[k, n]
      RKL_CUDA(launch_simt_gemm(dzf, 1, cw, a.as, H, 1, dW_s + size_t(cv0) * H, H, cw, static_cast<int>(H), n_rows,
                                0, n_dev, 2, s));
      // dHc[m, n] (+)= sum_k dz[m, k] W_s[cv0 + k, n]
      RKL_CUDA(launch_simt_gemm(dzf, cw, 1, a.bs + size_t(cv0) * H, H, 1, dHc, H, n_rows, static_cast<int>(H), cw,
                                c > 0, n_dev, 1, s));
    }
  }
  RKL_CUDA(launch_scatter_dh(dHc, row_idx, k_slot, N, n_dev, T, static_cast<int>(H), dH_s, s));
  return RKL_OK;
}

}  // namespace rkl

// ====================================================================== C ABI
using namespace rkl;

extern "C" {

#ifdef RKL_DEBUG
const char* rkl_version(void) { return "rkl 0.2 (sm_100a, debug bounds checks)"; }
#else
const char* rkl_version(void) { return "rkl 0.2 (sm_100a)"; }
#endif

const char* rkl_last_error(void) { return g_last_error.c_str(); }

// Workspace of the logits-pair mode: only the per-row constants of the backward.
static size_t pair_workspace_bytes(int64_t n_max) {
  const int64_t n = n_max < 1 ? 1 : n_max;
  const size_t n_pad = size_t(((n + 255) / 256) * 256);
  return 256 + align256(3 * n_pad * sizeof(float));
}

rkl_status rkl_workspace_size(rkl_payload payload, rkl_dtype dtype, int64_t n_max, int64_t B, int64_t Sm1, int64_t H,
                              int64_t V, size_t* bytes) {
  if (bytes == nullptr) return fail(RKL_ERR_NULL, "bytes is NULL");
  RKL_TRY(check_common(payload, dtype, B, Sm1, H, V, 0, 0));
  if (n_max < 0 || n_max > B * Sm1) return fail(RKL_ERR_SHAPE, "n_max outside [0, B*Sm1]");
  *bytes = payload == RKL_PAYLOAD_LOGITS_PAIR ? pair_workspace_bytes(n_max) : make_plan(payload, dtype, n_max, H, V).total;
  return RKL_OK;
}

rkl_status rkl_forward_logits_pair(const void* student_logits, const void* teacher_logits, rkl_dtype dtype, int64_t B,
                                   int64_t Sm1, int64_t V, const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                   rkl_reduction reduction, float* loss_tok, float* loss, float* saved,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  RKL_TRY(check_common(RKL_PAYLOAD_LOGITS_PAIR, dtype, B, Sm1, 64, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  RKL_TRY(check_ptr(student_logits, "student_logits"));
  RKL_TRY(check_ptr(teacher_logits, "teacher_logits"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(loss_tok, "loss_tok", false));
  RKL_TRY(check_ptr(loss, "loss", false));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(workspace, "workspace"));
  if (workspace_bytes < pair_workspace_bytes(N))
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, pair_workspace_bytes(N));
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = B * Sm1;
  RKL_CUDA(launch_pair_fwd(student_logits, teacher_logits, dtype == RKL_BF16, row_idx, N, n_dev, static_cast<int>(V),
                           saved, s));
  if (loss_tok) RKL_CUDA(launch_scatter_loss(saved, row_idx, N, n_dev, T, loss_tok, s));
  if (loss && reduction != RKL_REDUCE_NONE)
    RKL_CUDA(launch_reduce(saved, row_idx, N, n_dev, static_cast<int>(B), static_cast<int>(Sm1), reduction, loss, s));
  return RKL_OK;
}

rkl_status rkl_backward_logits_pair(const void* student_logits, const void* teacher_logits, rkl_dtype dtype,
                                    int64_t B, int64_t Sm1, int64_t V, const int32_t* row_idx, int32_t N,
                                    const int32_t* n_dev, rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok, void* dz, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  RKL_TRY(check_common(RKL_PAYLOAD_LOGITS_PAIR, dtype, B, Sm1, 64, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  RKL_TRY(check_ptr(student_logits, "student_logits"));
  RKL_TRY(check_ptr(teacher_logits, "teacher_logits"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(grad_loss, "grad_loss", false));
  RKL_TRY(check_ptr(grad_tok, "grad_tok", false));
  RKL_TRY(check_ptr(dz, "dz"));
  RKL_TRY(check_ptr(workspace, "workspace"));
  if (workspace_bytes < pair_workspace_bytes(N))
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, pair_workspace_bytes(N));
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = B * Sm1;
  const int64_t n = N < 1 ? 1 : N;
  const int n_pad = static_cast<int>(((n + 255) / 256) * 256);
  float* rowc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 256);
  if (N > 0)
    RKL_CUDA(launch_row_weights(saved, row_idx, N, n_dev, n_pad, static_cast<int>(B), static_cast<int>(Sm1),
                                reduction, grad_loss, grad_tok, rowc, nullptr, s));
  RKL_CUDA(launch_pair_bwd(student_logits, teacher_logits, dtype == RKL_BF16, row_idx, N, n_dev, n_pad, T,
                           static_cast<int>(V), rowc, dz, s));
  return RKL_OK;
}

// ---------------------------------------------------------------- top-k estimator
static rkl_status check_topk(const void* zs, const void* zt, rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t V,
                             const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                             const int32_t* targets, int reduction, void* workspace, size_t workspace_bytes) {
  RKL_TRY(check_common(RKL_PAYLOAD_LOGITS_PAIR, dtype, B, Sm1, 64, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  RKL_TRY(check_ptr(zs, "student_logits"));
  RKL_TRY(check_ptr(zt, "teacher_logits"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(targets, "targets"));
  RKL_TRY(check_ptr(workspace, "workspace"));
  if (k < 0) return fail(RKL_ERR_SHAPE, "k = %lld is negative", (long long)k);
  if (workspace_bytes < pair_workspace_bytes(N))
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, pair_workspace_bytes(N));
  return RKL_OK;
}

rkl_status rkl_forward_topk_pair(const void* student_logits, const void* teacher_logits, rkl_dtype dtype, int64_t B,
                                 int64_t Sm1, int64_t V, const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                 int64_t k, const int32_t* targets, rkl_reduction reduction, float* loss_tok,
                                 float* loss, float* saved, void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  RKL_TRY(check_topk(student_logits, teacher_logits, dtype, B, Sm1, V, row_idx, N, n_dev, k, targets, reduction,
                     workspace, workspace_bytes));
  RKL_TRY(check_ptr(loss_tok, "loss_tok", false));
  RKL_TRY(check_ptr(loss, "loss", false));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = B * Sm1;
  RKL_CUDA(launch_topk_fwd(student_logits, teacher_logits, dtype == RKL_BF16, row_idx, targets, N, n_dev, 0,
                           static_cast<int>(V), k, saved, saved + 3 * size_t(N), V, false, s));
  if (loss_tok) RKL_CUDA(launch_scatter_loss(saved, row_idx, N, n_dev, T, loss_tok, s));
  if (loss && reduction != RKL_REDUCE_NONE)
    RKL_CUDA(launch_reduce(saved, row_idx, N, n_dev, static_cast<int>(B), static_cast<int>(Sm1), reduction, loss, s));
  return RKL_OK;
}

rkl_status rkl_backward_topk_pair(const void* student_logits, const void* teacher_logits, rkl_dtype dtype,
                                  int64_t B, int64_t Sm1, int64_t V, const int32_t* row_idx, int32_t N,
                                  const int32_t* n_dev, const int32_t* targets, rkl_reduction reduction,
                                  const float* saved, const float* grad_loss, const float* grad_tok, void* dz,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  RKL_TRY(check_topk(student_logits, teacher_logits, dtype, B, Sm1, V, row_idx, N, n_dev, 0, targets, reduction,
                     workspace, workspace_bytes));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(grad_loss, "grad_loss", false));
  RKL_TRY(check_ptr(grad_tok, "grad_tok", false));
  RKL_TRY(check_ptr(dz, "dz"));
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = B * Sm1;
  const int64_t n = N < 1 ? 1 : N;
  const int n_pad = static_cast<int>(((n + 255) / 256) * 256);
  float* rowc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 256);
  if (N > 0)
    RKL_CUDA(launch_row_weights(saved, row_idx, N, n_dev, n_pad, static_cast<int>(B), static_cast<int>(Sm1),
                                reduction, grad_loss, grad_tok, rowc, nullptr, s));
  RKL_CUDA(launch_topk_bwd(student_logits, teacher_logits, dtype == RKL_BF16, row_idx, targets, N, n_dev, n_pad, T,
                           static_cast<int>(V), saved, N > 0 ? saved + 3 * size_t(N) : nullptr, rowc, dz, s));
  return RKL_OK;
}

// Top-k estimator on the hidden payload.  Forward: per block of up to
// kTopkBlockRows compacted rows, the tcgen05 kernel writes z_s and z_t (fp32)
// of the block, and the selection / estimate kernel of the logits-pair form
// runs on those rows.  Backward: the recompute + dz kernel with the top-k
// formula (membership from the same fp32 logits, bit for bit), then the
// gradient GEMMs of the exact path.
// Top-k forward of both tensor-core payloads.  Per block of up to
// kTopkBlockRows compacted rows, a tcgen05 kernel writes z_s and z_t (fp32)
// of the block -- on the hidden payload both by the tensor core, on the
// logits payload z_s by the tensor core and z_t copied (exactly) from the
// shipped bf16 teacher rows -- and the selection / estimate kernel of the
// logits-pair form runs on those rows.
static rkl_status forward_topk_impl(rkl_payload payload, const void* h_s, const void* teacher, const void* W_s,
                                    const void* W_t, rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                                    const int32_t* targets, rkl_reduction reduction, float* loss_tok, float* loss,
                                    float* saved, void* workspace, size_t workspace_bytes, void* stream) {
  const bool hidden = payload == RKL_PAYLOAD_TOPK_HIDDEN;
  RKL_TRY(check_common(payload, dtype, B, Sm1, H, V, N, reduction));
  RKL_TRY(check_n_dev(n_dev));
  if (dtype != RKL_BF16)
    return fail(RKL_ERR_UNSUPPORTED, "the top-k estimator on the tensor-core payloads needs bf16 inputs");
  if (k < 0) return fail(RKL_ERR_SHAPE, "k = %lld is negative", (long long)k);
  RKL_TRY(check_ptr(h_s, "h_s"));
  RKL_TRY(check_ptr(teacher, hidden ? "h_t" : "teacher_logits"));
  RKL_TRY(check_ptr(W_s, "W_s"));
  if (hidden) RKL_TRY(check_ptr(W_t, "W_t"));
  RKL_TRY(check_ptr(row_idx, "row_idx"));
  RKL_TRY(check_ptr(targets, "targets"));
  RKL_TRY(check_ptr(loss_tok, "loss_tok", false));
  RKL_TRY(check_ptr(loss, "loss", false));
  RKL_TRY(check_ptr(saved, "saved", N > 0));
  RKL_TRY(check_ptr(workspace, "workspace"));
  const Plan pl = make_plan(payload, dtype, N, H, V);
  if (workspace_bytes < pl.total)
    return fail(RKL_ERR_WORKSPACE, "workspace is %zu bytes, %zu needed", workspace_bytes, pl.total);
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = B * Sm1;
  if (N > 0) {
    const uint8_t* as = static_cast<const uint8_t*>(h_s);
    const uint8_t* at = hidden ? static_cast<const uint8_t*>(teacher) : nullptr;
    if (N < T || n_dev) {
      as = ws_at(workspace, pl.off_hcs);
      at = hidden ? ws_at(workspace, pl.off_hct) : nullptr;
      RKL_CUDA(launch_gather(h_s, hidden ? teacher : nullptr, const_cast<uint8_t*>(as), const_cast<uint8_t*>(at),
                             row_idx, nullptr, N, n_dev, static_cast<int>(H * 2), T, s));
    }
    float* zs = reinterpret_cast<float*>(ws_at(workspace, pl.off_z));
    float* zt = hidden ? zs + size_t(pl.zrows) * pl.zpitch : nullptr;
    for (int r0 = 0; r0 < N; r0 += pl.zrows) {
      const int nb = (N - r0) < pl.zrows ? (N - r0) : pl.zrows;
      FusedArgs a;
      memset(&a, 0, sizeof(a));
      RKL_TRY(make_map(&a.tm_as, as + size_t(r0) * H * 2, false, H, nb, H * 2, kBK, kBM));
      RKL_TRY(make_map(&a.tm_bs, W_s, false, H, V, H * 2, kBK, kFBN / 2));
      if (hidden) {
        RKL_TRY(make_map(&a.tm_at, at + size_t(r0) * H * 2, false, H, nb, H * 2, kBK, kBM));
        RKL_TRY(make_map(&a.tm_bt, W_t, false, H, V, H * 2, kBK, kFBN / 2));
      } else {
        // row p of the block is compacted row r0 + p: token row row_idx[r0 + p]
        a.teacher = static_cast<const uint16_t*>(teacher);
        a.teacher_rows = row_idx + r0;
        a.teacher_pitch = V;
      }
      RKL_TRY(make_map(&a.tm_zs, zs, true, V, nb, size_t(pl.zpitch) * 4, 32, 32));
      if (hidden) RKL_TRY(make_map(&a.tm_zt, zt, true, V, nb, size_t(pl.zpitch) * 4, 32, 32));
      a.N = nb;
      a.n_dev = n_dev;
      a.n_base = r0;
      a.n_pad = pl.n_pad;
      a.H = static_cast<int>(H);
      a.V = static_cast<int>(V);
      a.KB = static_cast<int>(H / kBK);
      a.IT = pl.VT;
      a.vt_base = 0;
      a.GT = 1;
      a.G = pl.VT;
      const int units = ((nb + 2 * kBM - 1) / (2 * kBM)) * a.G;  // at most
      RKL_CUDA(launch_fused_topk(1, hidden ? 2 : 1, a, 2 * units < sms ? 2 * units : sms, s));
      if (hidden)
        RKL_CUDA(launch_topk_fwd(zs, zt, false, row_idx + r0, targets, nb, n_dev, r0, static_cast<int>(V), k,
                                 saved + 3 * size_t(r0), saved + 3 * size_t(N) + 4 * size_t(r0), pl.zpitch, true, s));
      else
        RKL_CUDA(launch_topk_fwd_tlogits(zs, static_cast<const uint16_t*>(teacher), V, row_idx + r0, targets, nb,
                                         n_dev, r0, static_cast<int>(V), k, saved + 3 * size_t(r0),
                                         saved + 3 * size_t(N) + 4 * size_t(r0), pl.zpitch, s));
    }
  }
  if (loss_tok) RKL_CUDA(launch_scatter_loss(saved, row_idx, N, n_dev, T, loss_tok, s));
  if (loss && reduction != RKL_REDUCE_NONE)
    RKL_CUDA(launch_reduce(saved, row_idx, N, n_dev, static_cast<int>(B), static_cast<int>(Sm1), reduction, loss, s));
  return RKL_OK;
}

rkl_status rkl_forward_topk_hidden(const void* h_s, const void* h_t, const void* W_s, const void* W_t,
                                   rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                   const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                                   const int32_t* targets, rkl_reduction reduction, float* loss_tok, float* loss,
                                   float* saved, void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_topk_impl(RKL_PAYLOAD_TOPK_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, n_dev, k,
                           targets, reduction, loss_tok, loss, saved, workspace, workspace_bytes, stream);
}

rkl_status rkl_forward_topk_logits(const void* h_s, const void* W_s, const void* teacher_logits, rkl_dtype dtype,
                                   int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                                   const int32_t* n_dev, int64_t k, const int32_t* targets, rkl_reduction reduction,
                                   float* loss_tok, float* loss, float* saved, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_topk_impl(RKL_PAYLOAD_TOPK_LOGITS, h_s, teacher_logits, W_s, nullptr, dtype, B, Sm1, H, V, row_idx,
                           N, n_dev, k, targets, reduction, loss_tok, loss, saved, workspace, workspace_bytes, stream);
}

rkl_status rkl_backward_topk_logits(const void* h_s, const void* W_s, const void* teacher_logits, rkl_dtype dtype,
                                    int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                                    const int32_t* n_dev, const int32_t* targets, rkl_reduction reduction,
                                    const float* saved, const float* grad_loss, const float* grad_tok, float* dH_s,
                                    float* dW_s, void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return backward_impl(RKL_PAYLOAD_TOPK_LOGITS, h_s, teacher_logits, W_s, nullptr, dtype, B, Sm1, H, V, row_idx, N,
                       n_dev, reduction, saved, grad_loss, grad_tok, dH_s, dW_s, workspace, workspace_bytes, stream,
                       nullptr, targets);
}

rkl_status rkl_backward_topk_hidden(const void* h_s, const void* h_t, const void* W_s, const void* W_t,
                                    rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N, const int32_t* n_dev, const int32_t* targets,
                                    rkl_reduction reduction, const float* saved, const float* grad_loss,
                                    const float* grad_tok, float* dH_s, float* dW_s, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return backward_impl(RKL_PAYLOAD_TOPK_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, n_dev,
                       reduction, saved, grad_loss, grad_tok, dH_s, dW_s, workspace, workspace_bytes, stream, nullptr,
                       targets);
}

rkl_status rkl_compact_rows(const uint8_t* mask, int64_t B, int64_t Sm1, int32_t* row_idx, int32_t* n_dev,
                            void* stream) {
  RKL_NVTX_RANGE();
  if (mask == nullptr || row_idx == nullptr || n_dev == nullptr)
    return fail(RKL_ERR_NULL, "mask, row_idx and n_dev must be non-NULL");
  if (!aligned16(row_idx)) return fail(RKL_ERR_ALIGN, "row_idx is not 16-byte aligned");
  if (B < 1 || Sm1 < 1) return fail(RKL_ERR_SHAPE, "B and Sm1 must be >= 1");
  if (B * Sm1 >= (int64_t(1) << 31)) return fail(RKL_ERR_SHAPE, "B*Sm1 exceeds 2^31-1");
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  RKL_CUDA(launch_compact(mask, B * Sm1, row_idx, n_dev, static_cast<cudaStream_t>(stream)));
  return RKL_OK;
}

rkl_status rkl_forward_hidden(const void* h_s, const void* h_t, const void* W_s, const void* W_t, rkl_dtype dtype,
                              int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                              const int32_t* n_dev, rkl_reduction reduction, float* loss_tok, float* loss,
                              float* saved, void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_impl(RKL_PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, n_dev, reduction,
                      loss_tok, loss, saved, workspace, workspace_bytes, stream);
}

rkl_status rkl_forward_logits(const void* h_s, const void* W_s, const void* teacher_logits, rkl_dtype dtype,
                              int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                              const int32_t* n_dev, rkl_reduction reduction, float* loss_tok, float* loss,
                              float* saved, void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_impl(RKL_PAYLOAD_LOGITS, h_s, teacher_logits, W_s, nullptr, dtype, B, Sm1, H, V, row_idx, N, n_dev,
                      reduction, loss_tok, loss, saved, workspace, workspace_bytes, stream);
}

rkl_status rkl_forward_hidden_ex(const void* h_s, const void* h_t, const void* W_s, const void* W_t, rkl_dtype dtype,
                                 int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                                 const int32_t* n_dev, rkl_reduction reduction, float* loss_tok, float* loss,
                                 float* saved, const int32_t* targets, float* entropy, float* target_logprob,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_impl(RKL_PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, n_dev, reduction,
                      loss_tok, loss, saved, workspace, workspace_bytes, stream, false, targets, entropy,
                      target_logprob);
}

rkl_status rkl_forward_logits_ex(const void* h_s, const void* W_s, const void* teacher_logits, rkl_dtype dtype,
                                 int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx, int32_t N,
                                 const int32_t* n_dev, rkl_reduction reduction, float* loss_tok, float* loss,
                                 float* saved, const int32_t* targets, float* entropy, float* target_logprob,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return forward_impl(RKL_PAYLOAD_LOGITS, h_s, teacher_logits, W_s, nullptr, dtype, B, Sm1, H, V, row_idx, N, n_dev,
                      reduction, loss_tok, loss, saved, workspace, workspace_bytes, stream, false, targets, entropy,
                      target_logprob);
}

rkl_status rkl_backward(rkl_payload payload, const void* h_s, const void* teacher, const void* W_s, const void* W_t,
                        rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V, const int32_t* row_idx,
                        int32_t N, const int32_t* n_dev, rkl_reduction reduction, const float* saved,
                        const float* grad_loss, const float* grad_tok, float* dH_s, float* dW_s, void* workspace,
                        size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  return backward_impl(payload, h_s, teacher, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, n_dev, reduction, saved,
                       grad_loss, grad_tok, dH_s, dW_s, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- teacher per row
rkl_status rkl_compact_rows_multi(const uint8_t* mask, const int32_t* teacher_idx, int64_t B, int64_t Sm1,
                                  int32_t n_teachers, int32_t* row_idx, int32_t* n_dev, int32_t* counts,
                                  void* stream) {
  RKL_NVTX_RANGE();
  if (mask == nullptr || teacher_idx == nullptr || row_idx == nullptr || n_dev == nullptr || counts == nullptr)
    return fail(RKL_ERR_NULL, "mask, teacher_idx, row_idx, n_dev and counts must be non-NULL");
  if (!aligned16(row_idx) || !aligned16(teacher_idx))
    return fail(RKL_ERR_ALIGN, "row_idx and teacher_idx must be 16-byte aligned");
  if (B < 1 || Sm1 < 1) return fail(RKL_ERR_SHAPE, "B and Sm1 must be >= 1");
  if (B * Sm1 >= (int64_t(1) << 31)) return fail(RKL_ERR_SHAPE, "B*Sm1 exceeds 2^31-1");
  if (n_teachers < 1 || n_teachers > kMaxTeachers)
    return fail(RKL_ERR_SHAPE, "n_teachers = %d outside [1, %d]", n_teachers, kMaxTeachers);
  int sms = 0;
  RKL_TRY(device_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RKL_CUDA(cudaMemsetAsync(counts, 0, size_t(n_teachers + 1) * sizeof(int32_t), s));
  RKL_CUDA(launch_compact(mask, B * Sm1, row_idx, n_dev, s));
  RKL_CUDA(launch_count_teachers(mask, teacher_idx, B * Sm1, n_teachers, counts, s));
  return RKL_OK;
}

rkl_status rkl_workspace_size_multi(rkl_dtype dtype, int64_t n_max, int32_t n_teachers, int64_t B, int64_t Sm1,
                                    int64_t H, int64_t V, size_t* bytes) {
  if (bytes == nullptr) return fail(RKL_ERR_NULL, "bytes is NULL");
  RKL_TRY(check_common(RKL_PAYLOAD_HIDDEN, dtype, B, Sm1, H, V, 0, 0));
  if (n_max < 0 || n_max > B * Sm1) return fail(RKL_ERR_SHAPE, "n_max outside [0, B*Sm1]");
  if (n_teachers < 1 || n_teachers > kMaxTeachers)
    return fail(RKL_ERR_SHAPE, "n_teachers = %d outside [1, %d]", n_teachers, kMaxTeachers);
  *bytes = make_plan(RKL_PAYLOAD_HIDDEN, dtype, n_max, H, V, n_teachers).total;
  return RKL_OK;
}

rkl_status rkl_forward_hidden_multi(const void* h_s, const void* h_t, const void* W_s, const void* W_t,
                                   int32_t n_teachers, const int32_t* teacher_idx, const int32_t* counts,
                                   rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                   const int32_t* row_idx, int32_t N, rkl_reduction reduction, float* loss_tok,
                                   float* loss, float* saved, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  RKL_NVTX_RANGE();
  MultiTeacher mt;
  RKL_TRY(make_multi(n_teachers, teacher_idx, counts, N, &mt));
  return forward_impl(RKL_PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, nullptr, reduction,
                      loss_tok, loss, saved, workspace, workspace_bytes, stream, false, nullptr, nullptr, nullptr,
                      n_teachers > 1 ? &mt : nullptr);
}

rkl_status rkl_backward_hidden_multi(const void* h_s, const void* h_t, const void* W_s, const void* W_t,
                                    int32_t n_teachers, const int32_t* teacher_idx, const int32_t* counts,
                                    rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N, rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok, float* dH_s, float* dW_s,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  RKL_NVTX_RANGE();
  MultiTeacher mt;
  RKL_TRY(make_multi(n_teachers, teacher_idx, counts, N, &mt));
  return backward_impl(RKL_PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, nullptr, reduction,
                       saved, grad_loss, grad_tok, dH_s, dW_s, workspace, workspace_bytes, stream,
                       n_teachers > 1 ? &mt : nullptr);
}

rkl_status rkl_device_error(int32_t* code) {
  if (code == nullptr) return fail(RKL_ERR_NULL, "code is NULL");
  RKL_CUDA(cudaDeviceSynchronize());
  int v = 0, line_tc = 0, line_small = 0;
  RKL_CUDA(read_and_clear_device_error(&v));
  RKL_CUDA(read_and_clear_bounds_tc(&line_tc));
  RKL_CUDA(read_and_clear_bounds_small(&line_small));
  if (line_tc || line_small) v |= ERR_BOUNDS;
  *code = v;
  if (line_tc || line_small)
    return fail(RKL_ERR_DEVICE,
                "a bounds check failed (tc_kernels.cu line %d, small_kernels.cu line %d; 0 = none); the access was "
                "skipped and the outputs are invalid (bits 0x%x)",
                line_tc, line_small, v);
  if (v != 0) return fail(RKL_ERR_DEVICE, "a kernel wait ran out (bits 0x%x); its outputs are invalid", v);
  return RKL_OK;
}

int32_t rkl_kernel_count(void) { return K_COUNT; }

const char* rkl_kernel_name(int32_t kernel_id) { return kernel_name(kernel_id); }

rkl_status rkl_profile_enable(int32_t enable) {
  g_profile.store(enable != 0);
  return RKL_OK;
}

static rkl_status drain_profile() {
  std::vector<ProfRec> pend;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    pend.swap(g_prof_pending);
  }
  for (const ProfRec& r : pend) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
    if (e != cudaSuccess) return fail(RKL_ERR_CUDA, "profile event: %s", cudaGetErrorString(e));
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_ms[r.id] += ms;
    g_prof_n[r.id] += 1;
  }
  return RKL_OK;
}

rkl_status rkl_profile_reset(void) {
  RKL_TRY(drain_profile());
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int i = 0; i < K_COUNT; ++i) {
    g_prof_ms[i] = 0.0;
    g_prof_n[i] = 0;
  }
  return RKL_OK;
}

rkl_status rkl_profile_read(int32_t kernel_id, double* total_ms, int64_t* launches) {
  if (kernel_id < 0 || kernel_id >= K_COUNT) return fail(RKL_ERR_SHAPE, "kernel id %d out of range", kernel_id);
  if (total_ms == nullptr || launches == nullptr) return fail(RKL_ERR_NULL, "outputs are NULL");
  RKL_TRY(drain_profile());
  std::lock_guard<std::mutex> lk(g_prof_mu);
  *total_ms = g_prof_ms[kernel_id];
  *launches = g_prof_n[kernel_id];
  return RKL_OK;
}

int64_t rkl_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ====================================================================== no-allocation forward
// Scratch of rkl_forward_hidden_noalloc: one array in the library's device
// image.  Every GPU on which the library's kernels are loaded holds these
// bytes until the process exits, whether or not it ever calls that entry
// point.  Host code only sees a stand-in symbol for it; the device address is
// looked up per device below.
namespace rkl {
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

static std::mutex g_static_mu;
static void* g_static_ptr[64];  // device address of g_static_scratch, per device

// Looks up (once per device, with that device current) the device address of
// the static scratch array.
static rkl_status static_scratch_ptr(void** out) {
  int dev = 0;
  RKL_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RKL_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(RKL_ERR_CUDA, "cudaGetSymbolAddress(static scratch) failed on device %d: %s", dev,
                  cudaGetErrorString(e));
    g_static_ptr[dev] = ptr;
  }
  *out = g_static_ptr[dev];
  return RKL_OK;
}
}  // namespace rkl

extern "C" rkl_status rkl_forward_hidden_noalloc(const void* h_s, const void* h_t, const void* W_s, const void* W_t,
                                                 rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                                 const int32_t* row_idx, int32_t N, rkl_reduction reduction,
                                                 float* loss_tok, float* loss, float* saved, void* stream) {
  RKL_NVTX_RANGE();
  // Size check first, from the same layout the workspace path uses; nothing
  // on the device is touched when the problem does not fit.
  RKL_TRY(check_common(RKL_PAYLOAD_HIDDEN, dtype, B, Sm1, H, V, N, reduction));
  const Plan pl = make_plan(RKL_PAYLOAD_HIDDEN, dtype, N, H, V);
  if (pl.off_dz > kStaticScratchBytes)
    return fail(RKL_ERR_WORKSPACE,
                "rkl_forward_hidden_noalloc: this problem needs %zu bytes of scratch, the static limit is %zu "
                "bytes (%zu MiB); use rkl_forward_hidden with a caller workspace",
                pl.off_dz, kStaticScratchBytes, kStaticScratchBytes >> 20);
  void* scratch = nullptr;
  RKL_TRY(static_scratch_ptr(&scratch));
  // Every region of the scratch that the forward reads is written earlier in
  // the same call, so nothing needs clearing between calls.
  return forward_impl(RKL_PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, dtype, B, Sm1, H, V, row_idx, N, nullptr, reduction,
                      loss_tok, loss, saved, scratch, kStaticScratchBytes, stream, /*forward_only_workspace=*/true);
}
