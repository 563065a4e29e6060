// gdn_api.cu -- host side of libgdn.so: argument validation, workspace layout and the
// launch sequence of the prefill and decode paths.  Declarations and the contract of each
// entry point are in include/gdn.h.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>
#include <utility>

#include "gdn.h"
#include "gdn_common.cuh"
#include "k_chunk_simt.cuh"
#include "k_chunk_tc.cuh"
#include "k_decode.cuh"
#include "k_decode_multi.cuh"
#include "k_proj.cuh"
#include "k_bwd.cuh"
#include "k_stream.cuh"

using namespace gdn;

namespace {

__device__ float g_selftest_out[2];

constexpr int kVersion = 200;  // 0.2.0: the prefill-to-decode hand-off calls

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Path options (gdn_set_options).  The bf16-input prefill runs its chunk contractions on
// tcgen05 (bf16 hi/lo products); the fp32-input prefill keeps true fp32 FFMA.  The options
// select the slower alternatives for comparisons: bf16 inputs down the fp32 path, the output
// norm of the bf16 path in its own kernel, and plain stream order between the prefill kernels.
// Their initial value is read from the environment once per process (GDN_FORCE_SIMT=1,
// GDN_NO_FUSED_NORM=1, GDN_NO_PDL=1); later calls only read the word.
int env_flag(const char* name, const char* on) {
  const char* f = getenv(name);
  return f && strcmp(f, on) == 0 ? 1 : 0;
}
uint32_t options_from_env() {
  return (env_flag("GDN_FORCE_SIMT", "1") ? GDN_OPT_FORCE_FP32_PATH : 0u) |
         (env_flag("GDN_NO_FUSED_NORM", "1") ? GDN_OPT_SEPARATE_NORM : 0u) |
         (env_flag("GDN_NO_PDL", "1") ? GDN_OPT_NO_PDL : 0u);
}
std::atomic<uint32_t>& options_word() {
  static std::atomic<uint32_t> w{options_from_env()};
  return w;
}
bool opt(uint32_t bit) { return (options_word().load(std::memory_order_relaxed) & bit) != 0; }

bool use_tc(const gdn_dims_t* d) {
  if (d->in_dtype != GDN_DTYPE_BF16) return false;
  return !opt(GDN_OPT_FORCE_FP32_PATH);
}

// Workspace of the prefill, carved from the caller's buffer in this order.
struct WsLayout {
  size_t tab, seqc0, order, qn, kn, vc, g, beta, gam, W, Up, mqk, yraw, total;
  size_t kq, tp, gb, vs;  // tensor-core path
  int max_chunks;
  bool tc;
};

WsLayout ws_layout_tc(const gdn_dims_t* d) {
  WsLayout L{};
  L.tc = true;
  const size_t T = (size_t)d->total_tokens, hq = (size_t)d->h_qk, hv = (size_t)d->h_v;
  const size_t N = (size_t)d->n_seqs;
  L.max_chunks = (int)((T + CH - 1) / CH + N);
  const size_t MC = (size_t)L.max_chunks;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.tab = take(MC * sizeof(ChunkEntry));
  L.seqc0 = take((N + 1) * sizeof(int));
  L.order = take(N * sizeof(int));
  L.kq = take(MC * hq * KQ_BYTES);
  L.tp = take(MC * hv * TP_BYTES);
  L.gb = take(MC * hv * GB_FLOATS * 4);
  L.vs = take(MC * hv * VS_BYTES);
  L.yraw = take(T * hv * D * 4);
  L.total = off;
  return L;
}

WsLayout ws_layout(const gdn_dims_t* d) {
  if (use_tc(d)) return ws_layout_tc(d);
  WsLayout L{};
  const size_t T = (size_t)d->total_tokens, hq = (size_t)d->h_qk, hv = (size_t)d->h_v;
  const size_t N = (size_t)d->n_seqs;
  // every sequence contributes ceil(len / 64) <= len / 64 + 1 chunks
  L.max_chunks = (int)((T + CH - 1) / CH + N);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.tab = take((size_t)L.max_chunks * sizeof(ChunkEntry));
  L.seqc0 = take((N + 1) * sizeof(int));
  L.qn = take(T * hq * D * 4);
  L.kn = take(T * hq * D * 4);
  L.vc = take(T * hv * D * 4);
  L.g = take(T * hv * 4);
  L.beta = take(T * hv * 4);
  L.gam = take(T * hv * 8);  // gamma in fp64
  L.W = take(T * hv * D * 4);
  L.Up = take(T * hv * D * 4);
  L.mqk = take(T * hv * CH * 4);
  L.yraw = take(T * hv * D * 4);
  L.total = off;
  return L;
}

// ---- optional per-kernel event timing (gdn_profile_enable / gdn_profile_read) ----------
constexpr int kProfMax = 8192;
struct Prof {
  bool on = false;
  bool created = false;
  int n = 0;
  cudaEvent_t ev[2 * kProfMax];
  const char* name[kProfMax];
};
Prof g_prof;

int prof_begin(const char* name, cudaStream_t s) {
  if (!g_prof.on || g_prof.n >= kProfMax) return -1;
  const int i = g_prof.n++;
  g_prof.name[i] = name;
  cudaEventRecord(g_prof.ev[2 * i], s);
  return i;
}
void prof_end(int i, cudaStream_t s) {
  if (i >= 0) cudaEventRecord(g_prof.ev[2 * i + 1], s);
}
struct ProfScope {
  int i;
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t st) : i(prof_begin(name, st)), s(st) {}
  ~ProfScope() { prof_end(i, s); }
};

// Launches a tensor-core prefill kernel with programmatic dependent launch: its CTAs may
// become resident while the previous kernel on the stream drains, and wait in
// griddepcontrol.wait (their first statement) until it has completed, unless the options ask for plain
// stream order (option GDN_OPT_NO_PDL).  cluster_x > 1 adds a (cluster_x, 1, 1) cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (!opt(GDN_OPT_NO_PDL)) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const gdn_dims_t* d, bool decode) {
  if (!d) return GDN_ERR_NULL;
  if (d->n_seqs < 1 || d->total_tokens < 0 || d->h_qk < 1 || d->h_v < 1) return GDN_ERR_SHAPE;
  if (d->h_v % d->h_qk != 0 || d->h_v / d->h_qk > 8) return GDN_ERR_SHAPE;
  if (d->d_k != D || d->d_v != D) return GDN_ERR_SHAPE;
  if (2 * d->h_qk + d->h_v > 65535 || d->h_v > 65535) return GDN_ERR_SHAPE;
  if (decode && d->total_tokens != d->n_seqs) return GDN_ERR_SHAPE;
  if ((int64_t)d->total_tokens / CH + d->n_seqs + 1 > INT32_MAX) return GDN_ERR_SHAPE;
  // chunk slots index grid.y of the tensor-core kernels
  if (!decode && d->in_dtype == GDN_DTYPE_BF16 && (int64_t)d->total_tokens / CH + d->n_seqs + 1 > 65535)
    return GDN_ERR_SHAPE;
  if (!isfinite(d->q_scale) || !(d->l2_eps >= 0.0f) || !(d->rms_eps >= 0.0f)) return GDN_ERR_SHAPE;
  if ((d->in_dtype != GDN_DTYPE_F32 && d->in_dtype != GDN_DTYPE_BF16) ||
      (d->out_dtype != GDN_DTYPE_F32 && d->out_dtype != GDN_DTYPE_BF16))
    return GDN_ERR_DTYPE;
  return GDN_OK;
}

Dims kdims(const gdn_dims_t* d) {
  Dims k;
  k.n_seqs = d->n_seqs;
  k.total_tokens = d->total_tokens;
  k.h_qk = d->h_qk;
  k.h_v = d->h_v;
  k.in_bf16 = d->in_dtype == GDN_DTYPE_BF16;
  k.out_bf16 = d->out_dtype == GDN_DTYPE_BF16;
  k.q_scale = d->q_scale;
  k.l2_eps = d->l2_eps;
  k.rms_eps = d->rms_eps;
  return k;
}

int g_num_sms = 148;  // SM count of the current device (set by configure_device)

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
  if (f) return f;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !p)
    return nullptr;
  f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  fn.store(f);
  return f;
}

// Tensor map of a bf16 stream [T][nheads][128] whose box is 128 channels x box_heads heads x
// box_rows tokens (elements outside the tensor read as zeros).
int make_stream_map(CUtensorMap* m, const void* x, int T, int nheads, int box_heads, int box_rows) {
  memset(m, 0, sizeof(*m));
  PFN_cuTensorMapEncodeTiled_v12000 f = encode_tiled();
  if (!f) return GDN_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)nheads, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)nheads * D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GDN_OK : GDN_ERR_CUDA;
}

// Tensor map of a K-major bf16 matrix [rows][K] for the projection GEMM: boxes of 64 K x box_rows
// rows in the 128-byte swizzled layout (rows past the matrix read as zeros).
int make_kmajor_map(CUtensorMap* m, const void* x, long long rows, int K, int box_rows) {
  memset(m, 0, sizeof(*m));
  PFN_cuTensorMapEncodeTiled_v12000 f = encode_tiled();
  if (!f) return GDN_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)PJ_BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GDN_OK : GDN_ERR_CUDA;
}

// Opt the large-shared-memory kernels in once per device.
int configure_device() {
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  {
    int nsm = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return GDN_ERR_CUDA;
    g_num_sms = nsm > 0 ? nsm : 148;
  }
  if (done_mask.load() & bit) return GDN_OK;
  if (cudaFuncSetAttribute(k_phaseA_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PA_SMEM) !=
          cudaSuccess ||
      cudaFuncSetAttribute(k_phaseB_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PB_SMEM) !=
          cudaSuccess ||
      cudaFuncSetAttribute(k_chunkprep_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PA_TC_SMEM) !=
          cudaSuccess ||
      cudaFuncSetAttribute(k_chunkscan_tc<PB_Y_RAW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)PB_TC_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_chunkscan_tc<PB_Y_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)PB_TC_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_chunkscan_tc<PB_Y_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)PB_TC_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_proj_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PJ_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BW_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_decode_multi<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)DECM_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_decode_multi<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)DECM_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_decode_multi<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)DECM_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_decode_multi<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)DECM_SMEM) != cudaSuccess)
    return GDN_ERR_CUDA;
  done_mask.fetch_or(bit);
  return GDN_OK;
}

// Clusters of four phase-B CTAs (the slices of one value head) that fit on the device at
// once, per device; 0 if the query failed (then the fused output norm is not used).
int scan_clusters_per_wave() {
  static int cached[64];
  static std::atomic<uint64_t> known{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const uint64_t bit = 1ull << (dev & 63);
  if (known.load() & bit) return cached[dev & 63];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(D / TC_NV);
  cfg.blockDim = dim3(384);
  cfg.dynamicSmemBytes = PB_TC_SMEM;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = D / TC_NV;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_chunkscan_tc<PB_Y_BF16>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cached[dev & 63] = n;
  known.fetch_or(bit);
  return n;
}

template <bool IN_BF16>
void launch_prologue(const Dims& kd, int max_chunks, const ChunkEntry* tab, const void* q,
                     const void* k, const void* v, const float* a, const float* b,
                     const float* A_log, const float* dt_bias, const float* conv_w, float* qn,
                     float* kn, float* vc, float* g, float* beta, cudaStream_t s) {
  dim3 grid(max_chunks, 2 * kd.h_qk + kd.h_v);
  k_prologue<IN_BF16><<<grid, 256, 0, s>>>(kd, tab, q, k, v, a, b, A_log, dt_bias, conv_w, qn, kn,
                                           vc, g, beta);
}

void launch_epilogue(const Dims& kd, const float* yraw, const void* z, const float* norm_w, void* y,
                     cudaStream_t s) {
  const long rows = (long)kd.total_tokens * kd.h_v;
  const unsigned blocks = (unsigned)((rows + 8 * EPI_ROWS - 1) / (8 * EPI_ROWS));
  if (kd.in_bf16 && kd.out_bf16) k_epilogue<true, true><<<blocks, 256, 0, s>>>(kd, yraw, z, norm_w, y, rows);
  else if (kd.in_bf16) k_epilogue<true, false><<<blocks, 256, 0, s>>>(kd, yraw, z, norm_w, y, rows);
  else if (kd.out_bf16) k_epilogue<false, true><<<blocks, 256, 0, s>>>(kd, yraw, z, norm_w, y, rows);
  else k_epilogue<false, false><<<blocks, 256, 0, s>>>(kd, yraw, z, norm_w, y, rows);
}

}  // namespace

extern "C" {

int gdn_version(void) { return kVersion; }

uint32_t gdn_set_options(uint32_t flags) { return options_word().exchange(flags & GDN_OPT_ALL); }

uint32_t gdn_get_options(void) { return options_word().load(); }

const char* gdn_status_string(int code) {
  switch (code) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_NULL: return "GDN_ERR_NULL";
    case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE";
    case GDN_ERR_DTYPE: return "GDN_ERR_DTYPE";
    case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT";
    case GDN_ERR_INDEX: return "GDN_ERR_INDEX";
    default: return "GDN_ERR_UNKNOWN";
  }
}

size_t gdn_prefill_workspace_size(const gdn_dims_t* d) {
  if (check_dims(d, false) != GDN_OK) return 0;
  return ws_layout(d).total;
}

int gdn_prefill(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
                const float* a, const float* b, const float* A_log, const float* dt_bias,
                const float* conv_w, const float* norm_w, const float* init_state,
                const int32_t* cu_seqlens, void* y, float* final_state, void* workspace,
                size_t workspace_bytes, gdn_stream_t stream) {
  int rc = check_dims(d, false);
  if (rc != GDN_OK) return rc;
  if (!final_state || !A_log || !dt_bias || !conv_w || !norm_w) return GDN_ERR_NULL;
  if (d->total_tokens > 0 && (!q || !k || !v || !z || !a || !b || !y)) return GDN_ERR_NULL;
  if (!cu_seqlens && d->n_seqs != 1) return GDN_ERR_NULL;
  const void* ptrs[] = {q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, init_state, cu_seqlens,
                        y, final_state, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_ALIGN;
  const WsLayout L = ws_layout(d);
  if (!workspace || workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
  rc = configure_device();
  if (rc != GDN_OK) return rc;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  ChunkEntry* tab = reinterpret_cast<ChunkEntry*>(ws + L.tab);
  int* seqc0 = reinterpret_cast<int*>(ws + L.seqc0);
  const Dims kd = kdims(d);

  // One sequence without cu_seqlens: the tensor-core kernels compute the trivial tile map
  // themselves (no table, no launch).
  const bool need_map = !L.tc || cu_seqlens != nullptr;
  if (need_map) {
    ProfScope p("tilemap", s);
    k_tilemap<<<1, 1024, 0, s>>>(cu_seqlens, d->n_seqs, d->total_tokens, L.max_chunks, tab, seqc0,
                                 L.tc ? reinterpret_cast<int*>(ws + L.order) : nullptr);
  }
  if (L.tc) {
    const ChunkEntry* tabc = need_map ? tab : nullptr;
    const int* seqc0c = need_map ? seqc0 : nullptr;
    uint8_t* kq = reinterpret_cast<uint8_t*>(ws + L.kq);
    uint8_t* tp = reinterpret_cast<uint8_t*>(ws + L.tp);
    if (d->total_tokens > 0) {
      ProfScope p("chunk_prep_tc", s);
      // raw rows of a chunk with its conv history: one head of q or k, a pair of value heads
      CUtensorMap tm_q, tm_k, tm_v;
      if (make_stream_map(&tm_q, q, d->total_tokens, d->h_qk, 1, PF_ROWS) != GDN_OK ||
          make_stream_map(&tm_k, k, d->total_tokens, d->h_qk, 1, PF_ROWS) != GDN_OK ||
          make_stream_map(&tm_v, v, d->total_tokens, d->h_v, 2, PF_ROWS) != GDN_OK)
        return GDN_ERR_CUDA;
      if (launch_dep(k_chunkprep_tc, dim3(d->h_qk, L.max_chunks), dim3(256), PA_TC_SMEM, s, 1, kd, tabc, tm_q, tm_k,
                     tm_v, conv_w, a, b, A_log, dt_bias, kq, F(L.vs), tp, F(L.gb)) != cudaSuccess)
        return GDN_ERR_CUDA;
    }
    // The output norm runs inside phase B (clusters of the four slices of a head) unless that
    // would take more waves of CTAs than the unclustered launch.
    const long units = (long)d->n_seqs * d->h_v;
    const int per_wave = scan_clusters_per_wave();
    const long waves_fused = per_wave > 0 ? (units + per_wave - 1) / per_wave : 0;
    const long waves_plain = (units * (D / TC_NV) + g_num_sms - 1) / g_num_sms;
    const bool fused = per_wave > 0 && waves_fused <= waves_plain && !opt(GDN_OPT_SEPARATE_NORM);
    // one CTA per (sequence, value head, slice), flattened slice-fastest and sequence-slowest
    // in the order the tile map chose (longest sequence first)
    const long long nblk = (long long)d->n_seqs * d->h_v * (D / TC_NV);
    if (nblk > INT32_MAX) return GDN_ERR_SHAPE;
    const dim3 grid((unsigned)nblk);
    const int* order = need_map ? reinterpret_cast<const int*>(ws + L.order) : nullptr;
    if (fused) {
      ProfScope p("chunk_scan_tc_norm", s);
      const uint16_t* zb = static_cast<const uint16_t*>(z);
      cudaError_t e = launch_dep(kd.out_bf16 ? k_chunkscan_tc<PB_Y_BF16> : k_chunkscan_tc<PB_Y_F32>, grid, dim3(384),
                                 PB_TC_SMEM, s, D / TC_NV, kd, (const int*)cu_seqlens, seqc0c, order, (const uint8_t*)kq,
                                 (const uint8_t*)tp, (const float*)F(L.gb), (const float*)F(L.vs), init_state,
                                 F(L.yraw), final_state, zb, norm_w, y);
      if (e != cudaSuccess) return GDN_ERR_CUDA;
      return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    {
      ProfScope p("chunk_scan_tc", s);
      if (launch_dep(k_chunkscan_tc<PB_Y_RAW>, grid, dim3(288), PB_TC_SMEM, s, 1, kd, (const int*)cu_seqlens, seqc0c,
                     order, (const uint8_t*)kq, (const uint8_t*)tp, (const float*)F(L.gb), (const float*)F(L.vs),
                     init_state, F(L.yraw), final_state, (const uint16_t*)nullptr, (const float*)nullptr,
                     (void*)nullptr) != cudaSuccess)
        return GDN_ERR_CUDA;
    }
    if (d->total_tokens > 0) {
      ProfScope p("epilogue", s);
      launch_epilogue(kd, F(L.yraw), z, norm_w, y, s);
    }
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }
  if (d->total_tokens > 0) {
    {
      ProfScope p("prologue", s);
      if (kd.in_bf16)
        launch_prologue<true>(kd, L.max_chunks, tab, q, k, v, a, b, A_log, dt_bias, conv_w, F(L.qn),
                              F(L.kn), F(L.vc), F(L.g), F(L.beta), s);
      else
        launch_prologue<false>(kd, L.max_chunks, tab, q, k, v, a, b, A_log, dt_bias, conv_w, F(L.qn),
                               F(L.kn), F(L.vc), F(L.g), F(L.beta), s);
    }
    ProfScope p("chunk_phaseA_simt", s);
    k_phaseA_simt<<<dim3(L.max_chunks, d->h_v), 256, PA_SMEM, s>>>(
        kd, tab, F(L.qn), F(L.kn), F(L.vc), F(L.g), F(L.beta), reinterpret_cast<double*>(ws + L.gam), F(L.W),
        F(L.Up), F(L.mqk));
  }
  {
    ProfScope p("chunk_phaseB_simt", s);
    k_phaseB_simt<<<dim3(d->n_seqs, d->h_v, D / PB_VS), 256, PB_SMEM, s>>>(
        kd, cu_seqlens, F(L.qn), F(L.kn), reinterpret_cast<const double*>(ws + L.gam), F(L.W), F(L.Up), F(L.mqk), init_state, F(L.yraw),
        final_state);
  }
  if (d->total_tokens > 0) {
    ProfScope p("epilogue", s);
    launch_epilogue(kd, F(L.yraw), z, norm_w, y, s);
  }
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// One decode step, on per-sequence state (slots == nullptr) or on pool slots.
static int decode_impl(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
                const float* a, const float* b, const float* A_log, const float* dt_bias,
                const float* conv_w, const float* norm_w, void* conv_state, float* state, void* y,
                const int32_t* slots, int n_slots, gdn_stream_t stream) {
  int rc = check_dims(d, true);
  if (rc != GDN_OK) return rc;
  const void* ptrs[] = {q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, y};
  for (const void* p : ptrs)
    if (!p) return GDN_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  if (d->h_qk > 65535) return GDN_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Dims kd = kdims(d);
  dim3 grid(d->n_seqs, d->h_qk);
  ProfScope p("decode", s);
  if (kd.in_bf16 && kd.out_bf16)
    k_decode<true, true><<<grid, 256, 0, s>>>(kd, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w,
                                              conv_state, state, y, slots, n_slots);
  else if (kd.in_bf16)
    k_decode<true, false><<<grid, 256, 0, s>>>(kd, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w,
                                               conv_state, state, y, slots, n_slots);
  else if (kd.out_bf16)
    k_decode<false, true><<<grid, 256, 0, s>>>(kd, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w,
                                               conv_state, state, y, slots, n_slots);
  else
    k_decode<false, false><<<grid, 256, 0, s>>>(kd, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w,
                                                conv_state, state, y, slots, n_slots);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_decode(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
               const float* a, const float* b, const float* A_log, const float* dt_bias,
               const float* conv_w, const float* norm_w, void* conv_state, float* state, void* y,
               gdn_stream_t stream) {
  return decode_impl(d, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, y, nullptr, 0,
                     stream);
}

int gdn_decode_slots(const gdn_dims_t* d, const void* q, const void* k, const void* v, const void* z,
                     const float* a, const float* b, const float* A_log, const float* dt_bias,
                     const float* conv_w, const float* norm_w, void* conv_state_pool, float* state_pool,
                     int32_t n_slots, const int32_t* slot_ids, void* y, gdn_stream_t stream) {
  if (!slot_ids) return GDN_ERR_NULL;
  if (!aligned16(slot_ids)) return GDN_ERR_ALIGN;
  if (n_slots < 1) return GDN_ERR_SHAPE;
  return decode_impl(d, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state_pool, state_pool, y,
                     slot_ids, n_slots, stream);
}

int gdn_decode_multi(const gdn_dims_t* d, int32_t n_tokens, const void* q, const void* k, const void* v,
                     const void* z, const float* a, const float* b, const float* A_log, const float* dt_bias,
                     const float* conv_w, const float* norm_w, void* conv_state, float* state, void* y,
                     gdn_stream_t stream) {
  if (!d) return GDN_ERR_NULL;
  if (n_tokens < 1 || n_tokens > DECM_KMAX) return GDN_ERR_SHAPE;
  if ((int64_t)d->n_seqs * n_tokens != (int64_t)d->total_tokens) return GDN_ERR_SHAPE;
  gdn_dims_t d1 = *d;
  d1.total_tokens = d->n_seqs;  // one entry per sequence, n_tokens tokens each
  // One token per sequence is a plain decode step (same layouts): the single-token kernel,
  // which keeps eight rows of 32 lanes in flight per warp, is the faster one for it.
  if (n_tokens == 1)
    return decode_impl(&d1, q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, y, nullptr, 0,
                       stream);
  int rc = check_dims(&d1, true);
  if (rc != GDN_OK) return rc;
  const void* ptrs[] = {q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, y};
  for (const void* p : ptrs)
    if (!p) return GDN_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  if (d->h_qk > 65535) return GDN_ERR_SHAPE;
  rc = configure_device();
  if (rc != GDN_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Dims kd = kdims(&d1);
  const dim3 grid(d->n_seqs, d->h_qk);
  const size_t smem = decm_smem_bytes(n_tokens, d->h_v / d->h_qk);
  ProfScope p("decode_multi", s);
  if (kd.in_bf16 && kd.out_bf16)
    k_decode_multi<true, true><<<grid, 256, smem, s>>>(kd, n_tokens, q, k, v, z, a, b, A_log, dt_bias, conv_w,
                                                      norm_w, conv_state, state, y);
  else if (kd.in_bf16)
    k_decode_multi<true, false><<<grid, 256, smem, s>>>(kd, n_tokens, q, k, v, z, a, b, A_log, dt_bias, conv_w,
                                                       norm_w, conv_state, state, y);
  else if (kd.out_bf16)
    k_decode_multi<false, true><<<grid, 256, smem, s>>>(kd, n_tokens, q, k, v, z, a, b, A_log, dt_bias, conv_w,
                                                       norm_w, conv_state, state, y);
  else
    k_decode_multi<false, false><<<grid, 256, smem, s>>>(kd, n_tokens, q, k, v, z, a, b, A_log, dt_bias, conv_w,
                                                        norm_w, conv_state, state, y);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Workspace of the recurrence backward, carved from the caller's buffer in this order.
struct BwWs {
  size_t tab, seqc0, ck, part, total;
  int max_chunks;
};
BwWs bw_ws(const gdn_dims_t* d) {
  BwWs L{};
  const size_t T = (size_t)d->total_tokens, hv = (size_t)d->h_v, N = (size_t)d->n_seqs;
  L.max_chunks = (int)((T + CH - 1) / CH + N);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.tab = take((size_t)L.max_chunks * sizeof(ChunkEntry));
  L.seqc0 = take((N + 1) * sizeof(int));
  L.ck = take((size_t)L.max_chunks * hv * BW_CK_FLOATS * 4);
  L.part = take((size_t)BW_SL * T * hv * BW_RED * 4);
  L.total = off;
  return L;
}

// C = A B^T on tcgen05 into the output segments of `po` (M rows of A, N rows of B, K columns).
static int proj_launch(const void* A, long long M, const void* B, int N, int K, const ProjOut& po,
                       gdn_stream_t stream) {
  int rc = configure_device();
  if (rc != GDN_OK) return rc;
  if (M == 0) return GDN_OK;
  CUtensorMap ta, tb;
  if (make_kmajor_map(&ta, A, M, K, PJ_BM) != GDN_OK || make_kmajor_map(&tb, B, N, K, PJ_BN) != GDN_OK)
    return GDN_ERR_CUDA;
  const long long ntiles = ((M + PJ_BM - 1) / PJ_BM) * (long long)((N + PJ_BN - 1) / PJ_BN);
  if (ntiles > (1LL << 30)) return GDN_ERR_SHAPE;
  const unsigned grid = (unsigned)std::min<long long>(ntiles, g_num_sms);  // persistent: one CTA per SM
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("proj_gemm", s);
  k_proj_gemm<<<grid, 192, PJ_SMEM, s>>>((int)M, N, K, ta, tb, po);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_in_proj(const gdn_dims_t* d, int32_t hidden, const void* x, const void* w_in, void* q, void* k, void* v,
                void* z, float* a, float* b, gdn_stream_t stream) {
  int rc = check_dims(d, false);
  if (rc != GDN_OK) return rc;
  if (d->in_dtype != GDN_DTYPE_BF16) return GDN_ERR_DTYPE;
  if (hidden <= 0 || hidden % PJ_BK != 0 || hidden > (1 << 20)) return GDN_ERR_SHAPE;
  const void* ptrs[] = {x, w_in, q, k, v, z, a, b};
  for (const void* p : ptrs)
    if (!p) return GDN_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const int nq = d->h_qk * D, nv = d->h_v * D;
  const long long N = 2LL * nq + 2LL * nv + 2LL * d->h_v;
  if (N > (1 << 24)) return GDN_ERR_SHAPE;
  ProjOut po{};
  po.nseg = 6;
  int n = 0;
  auto seg = [&](int i, int width, long long ld, int f32, void* out) {
    po.seg[i].n0 = n;
    po.seg[i].n1 = n + width;
    po.seg[i].ld = ld;
    po.seg[i].f32 = f32;
    po.seg[i].out = out;
    n += width;
  };
  seg(0, nq, nq, 0, q);
  seg(1, nq, nq, 0, k);
  seg(2, nv, nv, 0, v);
  seg(3, nv, nv, 0, z);
  seg(4, d->h_v, d->h_v, 1, a);
  seg(5, d->h_v, d->h_v, 1, b);
  return proj_launch(x, d->total_tokens, w_in, (int)N, hidden, po, stream);
}

int gdn_out_proj(const gdn_dims_t* d, int32_t hidden, const void* y, const void* w_out, void* out,
                 gdn_stream_t stream) {
  int rc = check_dims(d, false);
  if (rc != GDN_OK) return rc;
  if (d->out_dtype != GDN_DTYPE_BF16) return GDN_ERR_DTYPE;
  if (hidden <= 0 || hidden % 32 != 0 || hidden > (1 << 20)) return GDN_ERR_SHAPE;
  const void* ptrs[] = {y, w_out, out};
  for (const void* p : ptrs)
    if (!p) return GDN_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const int K = d->h_v * D;
  ProjOut po{};
  po.nseg = 1;
  po.seg[0].n0 = 0;
  po.seg[0].n1 = hidden;
  po.seg[0].ld = hidden;
  po.seg[0].f32 = 0;
  po.seg[0].out = out;
  return proj_launch(y, d->total_tokens, w_out, hidden, K, po, stream);
}

// The backward runs in fp32 throughout: the dims' dtype codes are not read.
static int check_dims_bwd(const gdn_dims_t* d) {
  if (!d) return GDN_ERR_NULL;
  gdn_dims_t df = *d;
  df.in_dtype = GDN_DTYPE_F32;
  df.out_dtype = GDN_DTYPE_F32;
  return check_dims(&df, false);
}

size_t gdn_recurrence_backward_workspace_size(const gdn_dims_t* d) {
  if (check_dims_bwd(d) != GDN_OK) return 0;
  return bw_ws(d).total;
}

int gdn_recurrence_backward(const gdn_dims_t* d, const float* qh, const float* kh, const float* v, const float* g,
                            const float* beta, const float* init_state, const int32_t* cu_seqlens, const float* dy,
                            const float* dS_final, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                            float* dS_init, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  int rc = check_dims_bwd(d);
  if (rc != GDN_OK) return rc;
  if (!dS_init) return GDN_ERR_NULL;
  if (d->total_tokens > 0 && (!qh || !kh || !v || !g || !beta || !dy || !dq || !dk || !dv || !dg || !dbeta))
    return GDN_ERR_NULL;
  if (!cu_seqlens && d->n_seqs != 1) return GDN_ERR_NULL;
  const void* ptrs[] = {qh, kh, v, g, beta, init_state, cu_seqlens, dy, dS_final, dq, dk, dv, dg, dbeta, dS_init,
                        workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_ALIGN;
  const BwWs L = bw_ws(d);
  if (!workspace || workspace_bytes < L.total) return GDN_ERR_WORKSPACE;
  rc = configure_device();
  if (rc != GDN_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  ChunkEntry* tab = reinterpret_cast<ChunkEntry*>(ws + L.tab);
  int* seqc0 = reinterpret_cast<int*>(ws + L.seqc0);
  const Dims kd = kdims(d);
  if (cu_seqlens) {
    ProfScope p("tilemap", s);
    k_tilemap<<<1, 1024, 0, s>>>(cu_seqlens, d->n_seqs, d->total_tokens, L.max_chunks, tab, seqc0, nullptr);
  }
  {
    ProfScope p("recurrence_bwd", s);
    k_bwd<<<dim3(d->n_seqs, d->h_v, BW_SL), BW_THREADS, BW_SMEM, s>>>(
        kd, cu_seqlens, cu_seqlens ? seqc0 : nullptr, qh, kh, v, g, beta, init_state, dy, dS_final, dv, dS_init,
        F(L.ck), F(L.part));
  }
  if (d->total_tokens > 0) {
    ProfScope p("recurrence_bwd_sum", s);
    k_bwd_sum<<<dim3(d->total_tokens, d->h_qk), D, 0, s>>>(kd, F(L.part), g, dq, dk, dbeta, dg);
  }
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_prefill_conv_state(const gdn_dims_t* d, const void* q, const void* k, const void* v,
                           const int32_t* cu_seqlens, void* conv_state, gdn_stream_t stream) {
  const int rc = check_dims(d, false);
  if (rc != GDN_OK) return rc;
  if (!conv_state) return GDN_ERR_NULL;
  if (d->total_tokens > 0 && (!q || !k || !v)) return GDN_ERR_NULL;
  if (!cu_seqlens && d->n_seqs != 1) return GDN_ERR_NULL;
  const void* ptrs[] = {q, k, v, cu_seqlens, conv_state};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Dims kd = kdims(d);
  const dim3 grid(d->n_seqs, 3);
  ProfScope p("conv_state_out", s);
  if (kd.in_bf16)
    k_conv_state_out<uint16_t><<<grid, 256, 0, s>>>(kd, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                                    static_cast<const uint16_t*>(v), cu_seqlens,
                                                    static_cast<uint16_t*>(conv_state));
  else
    k_conv_state_out<float><<<grid, 256, 0, s>>>(kd, static_cast<const float*>(q), static_cast<const float*>(k),
                                                 static_cast<const float*>(v), cu_seqlens,
                                                 static_cast<float*>(conv_state));
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_profile_enable(int on) {
  if (on && !g_prof.created) {
    for (int i = 0; i < 2 * kProfMax; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return GDN_ERR_CUDA;
    g_prof.created = true;
  }
  g_prof.on = on != 0;
  return GDN_OK;
}

int gdn_profile_read(gdn_kernel_time_t* out, int max_entries) {
  if (!out) return GDN_ERR_NULL;
  int m = 0;
  for (int i = 0; i < g_prof.n; ++i) {
    float ms = 0.0f;
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess)
      return GDN_ERR_CUDA;
    int e = 0;
    while (e < m && strcmp(out[e].name, g_prof.name[i]) != 0) ++e;
    if (e == m) {
      if (m == max_entries) continue;
      out[m].name = g_prof.name[i];
      out[m].launches = 0;
      out[m].total_ms = 0.0;
      ++m;
    }
    out[e].launches += 1;
    out[e].total_ms += ms;
  }
  g_prof.n = 0;
  return m;
}

int gdn_selftest_tc(int case_id, float* out2) {
  if (!out2) return GDN_ERR_NULL;
  if (case_id < 0 || case_id > 5) return GDN_ERR_SHAPE;
  float zero[2] = {0.0f, 0.0f};
  if (cudaMemcpyToSymbol(g_selftest_out, zero, sizeof zero) != cudaSuccess) return GDN_ERR_CUDA;
  float* dptr = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&dptr), g_selftest_out) != cudaSuccess) return GDN_ERR_CUDA;
  const int smem = 160 * 1024;
  cudaError_t e = cudaSuccess;
  switch (case_id) {
    case 0:
      e = cudaFuncSetAttribute(k_selftest_umma<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<0><<<1, 128, smem>>>(dptr);
      break;
    case 1:
      e = cudaFuncSetAttribute(k_selftest_umma<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<1><<<1, 128, smem>>>(dptr);
      break;
    case 2:
      e = cudaFuncSetAttribute(k_selftest_umma<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<2><<<1, 128, smem>>>(dptr);
      break;
    case 3:
      e = cudaFuncSetAttribute(k_selftest_umma<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<3><<<1, 128, smem>>>(dptr);
      break;
    case 4:
      e = cudaFuncSetAttribute(k_selftest_umma<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<4><<<1, 128, smem>>>(dptr);
      break;
    default:
      e = cudaFuncSetAttribute(k_selftest_umma<5>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_selftest_umma<5><<<1, 128, smem>>>(dptr);
  }
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(out2, g_selftest_out, sizeof zero) != cudaSuccess) return GDN_ERR_CUDA;
  return GDN_OK;
}

int gdn_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return GDN_ERR_SHAPE;
  const unsigned long long v = ns;
  return cudaMemcpyToSymbol(g_gdn_wait_ns, &v, sizeof v) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_selftest_wait_timeout(gdn_stream_t stream) {
  k_selftest_wait_timeout<<<1, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

int gdn_read_device_status(gdn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GDN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gdn_status, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_gdn_status, &zero, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  return v;
}

}  // extern "C"
