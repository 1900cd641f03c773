// lynx_api.cu -- the C ABI of include/lynx.h: argument checks, workspace
// layout, TMA descriptor encoding, kernel launches, device status and the
// host-side metadata layout conversions.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "lynx.h"
#include "lynx_internal.h"

// Status words, one per stream: the first error code a kernel launched on the
// stream records wins.  Slot 0 is shared by the streams that find every other
// slot taken.
constexpr int kStatusSlots = 1024;
static __device__ uint32_t g_lynx_status_words[kStatusSlots];

// Scratch of lynx_sparsify_noalloc: per-split partial row sums, then s (when
// the caller gives no row_scale buffer).  Sized for LYNX_SPARSIFY_NOALLOC_MAX_ROWS.
constexpr size_t kNoAllocLpartBytes = size_t(8) * LYNX_SPARSIFY_NOALLOC_MAX_ROWS * 8;
constexpr size_t kNoAllocScratchBytes = kNoAllocLpartBytes + size_t(LYNX_SPARSIFY_NOALLOC_MAX_ROWS) * 4;
static __device__ __align__(256) unsigned char g_sparsify_noalloc_scratch[kNoAllocScratchBytes];

namespace lynx {

namespace {

constexpr int kMaxDevices = 64;

std::atomic<int> g_stall{0};
std::atomic<void*> g_split_event{nullptr};
std::atomic<int> g_profile_part{0};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

struct DeviceState {
  std::once_flag once;
  uint32_t* status = nullptr;  // device address of the status word array
  int sms = 0;
  cudaError_t err = cudaSuccess;
  std::mutex slots_mu;         // guards slot_of and next_slot
  std::unordered_map<uintptr_t, int> slot_of;
  int next_slot = 1;
};
DeviceState g_dev[kMaxDevices];

// Status word of `stream` (assigned on first use; slot 0 once all are taken).
// Kernels record their errors there and lynx_check_error(stream) reads it.
uint32_t* stream_status(DeviceState* ds, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(ds->slots_mu);
  const uintptr_t key = reinterpret_cast<uintptr_t>(stream);
  auto it = ds->slot_of.find(key);
  int slot = 0;
  if (it != ds->slot_of.end()) {
    slot = it->second;
  } else if (ds->next_slot < kStatusSlots) {
    slot = ds->next_slot++;
    ds->slot_of.emplace(key, slot);
  }
  return ds->status + slot;
}

// The slot of `stream` if it has one (-1 if nothing was ever launched on it).
int find_stream_slot(DeviceState* ds, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(ds->slots_mu);
  auto it = ds->slot_of.find(reinterpret_cast<uintptr_t>(stream));
  if (it != ds->slot_of.end()) return it->second;
  return ds->next_slot >= kStatusSlots ? 0 : -1;
}

// Streams and events of lynx_linear_host, made once per device: copies in and
// copies out run on their own streams so that they overlap each other (the link
// is full duplex) and the kernels on the caller's stream.
constexpr int kHostMaxChunks = 8;
struct HostPipe {
  std::once_flag once;
  std::mutex enqueue;  // one call's enqueue sequence at a time (events are reused)
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, out_done = nullptr;
  cudaEvent_t in_done[kHostMaxChunks] = {};
  cudaEvent_t comp_done[kHostMaxChunks] = {};
  cudaError_t err = cudaSuccess;
};
HostPipe g_host[kMaxDevices];

HostPipe* host_pipe() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  HostPipe& h = g_host[dev];
  std::call_once(h.once, [&h]() {
    auto ok = [&h](cudaError_t e) {
      if (h.err == cudaSuccess) h.err = e;
      return h.err == cudaSuccess;
    };
    ok(cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking));
    ok(cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking));
    ok(cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&h.out_done, cudaEventDisableTiming));
    for (int i = 0; i < kHostMaxChunks; ++i) {
      ok(cudaEventCreateWithFlags(&h.in_done[i], cudaEventDisableTiming));
      ok(cudaEventCreateWithFlags(&h.comp_done[i], cudaEventDisableTiming));
    }
  });
  return h.err == cudaSuccess ? &h : nullptr;
}

// Row chunks of lynx_linear_host: up to kHostMaxChunks, each a multiple of 256
// rows (the GEMM's CTA-pair row block) and, but for a single chunk, at least
// 512.  The copy of the last chunk back to the host is the part that nothing
// overlaps, so more, smaller chunks shorten it; the layer on a chunk runs well
// under the time of its copies.
int64_t host_chunk_rows(int64_t M) {
  int64_t n = M / 512;
  n = n < 1 ? 1 : (n > kHostMaxChunks ? kHostMaxChunks : n);
  const int64_t rows = (M + n - 1) / n;
  return ((rows + 255) / 256) * 256;
}

void resolve_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// Current device's state (status word address, SM count), set up once.
DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& d = g_dev[dev];
  std::call_once(d.once, [&d, dev]() {
    void* p = nullptr;
    d.err = cudaGetSymbolAddress(&p, g_lynx_status_words);
    if (d.err == cudaSuccess) d.status = static_cast<uint32_t*>(p);
    if (d.err == cudaSuccess) d.err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  });
  return d.err == cudaSuccess ? &d : nullptr;
}

// Device address of this device's noalloc scratch, looked up once per device.
struct NoAllocState {
  std::once_flag once;
  uint8_t* scratch = nullptr;
  cudaError_t err = cudaSuccess;
};
NoAllocState g_noalloc[kMaxDevices];

uint8_t* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  NoAllocState& st = g_noalloc[dev];
  std::call_once(st.once, [&st]() {
    void* p = nullptr;
    st.err = cudaGetSymbolAddress(&p, g_sparsify_noalloc_scratch);
    if (st.err == cudaSuccess) st.scratch = static_cast<uint8_t*>(p);
  });
  return st.err == cudaSuccess ? st.scratch : nullptr;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WorkspaceLayout {
  size_t vals, meta, scale, t, lpart, tpart, flags, total;
};

// lynx_linear's workspace: kept values | metadata | s | T (or T/s) | partials |
// one state word per 32-row slice (the GEMM's combining step)
WorkspaceLayout workspace_layout(int64_t M, int64_t K, int64_t r) {
  const size_t m = static_cast<size_t>(M);
  const size_t rr = static_cast<size_t>(r > 0 ? r : kLoraRankDefault);
  WorkspaceLayout w;
  w.vals = 0;
  w.meta = align256(w.vals + m * static_cast<size_t>(K));
  w.scale = align256(w.meta + lynx_meta_bytes(M, K));
  w.t = align256(w.scale + m * 4);
  w.lpart = align256(w.t + m * rr * 2);
  w.tpart = align256(w.lpart + static_cast<size_t>(kMaxSplit) * m * 8);
  w.flags = align256(w.tpart + static_cast<size_t>(kMaxSplit) * m * rr * 4);
  w.total = align256(w.flags + static_cast<size_t>(fin_slices(M)) * 4);
  return w;
}

// lynx_sparsify's workspace: partial sums | s (used when no row_scale is given)
struct SparsifyWorkspace {
  size_t lpart, scale, total;
};

SparsifyWorkspace sparsify_workspace(int64_t M) {
  const size_t m = static_cast<size_t>(M);
  SparsifyWorkspace w;
  w.lpart = 0;
  w.scale = align256(static_cast<size_t>(kMaxSplit) * m * 8);
  w.total = align256(w.scale + m * 4);
  return w;
}

lynx_status check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || K < 64 || K % 64 != 0) return LYNX_ERR_UNSUPPORTED_SHAPE;
  if (N != 0 && (N < 8 || N % 8 != 0)) return LYNX_ERR_UNSUPPORTED_SHAPE;
  // TMA coordinates are 32-bit; keep every extent comfortably inside
  if (M > (int64_t(1) << 30) || K > (int64_t(1) << 30) || N > (int64_t(1) << 30))
    return LYNX_ERR_UNSUPPORTED_SHAPE;
  return LYNX_OK;
}

bool rank_supported(int64_t r) {
  return r >= kLoraRankAlign && r <= kLoraRankMax && r % kLoraRankAlign == 0;
}

// A and B both given (then r is their rank) or both NULL (then r is 0 or any
// supported rank, which only sizes nothing)
lynx_status check_lora(const void* A, const void* B, int64_t r) {
  if ((A == nullptr) != (B == nullptr)) return LYNX_ERR_INVALID_ARG;
  if (A != nullptr && !rank_supported(r)) return LYNX_ERR_UNSUPPORTED_SHAPE;
  if (A == nullptr && r != 0 && !rank_supported(r)) return LYNX_ERR_UNSUPPORTED_SHAPE;
  return LYNX_OK;
}

lynx_status map_cuda(cudaError_t e) { return e == cudaSuccess ? LYNX_OK : LYNX_ERR_CUDA; }

int gemm_bn(int64_t N) { return N >= 1024 ? 256 : 128; }

// The pair GEMM combines the sparsify pass's partials itself (no finalize_kernel).
struct FusedFinalize {
  int mode = 0;  // 1: s and (with LoRA) bf16(T / s); 2: bf16(T)
  int split = 1;
  const float2* lpart = nullptr;
  const float* tpart = nullptr;
  float* scale = nullptr;
  void* t = nullptr;
  uint32_t* flags = nullptr;  // one state word per 32-row slice
};

lynx_status run_sparsify(DeviceState* ds, const void* X, const void* A, int64_t M, int64_t K,
                         int64_t r, void* vals, void* meta, float* row_scale, void* t_out,
                         float2* lpart, float* tpart, int mode, cudaStream_t stream,
                         const FusedFinalize* fin = nullptr) {
  SparsifyLaunch p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_bf16_2d(&p.tm_x, X, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return LYNX_ERR_CUDA;
  if (mode & kModeLora) {
    if (!encode_bf16_2d(&p.tm_a, A, K, r, K * 2, 64, static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B))
      return LYNX_ERR_CUDA;
  }
  if ((mode & kModeSelect) && !(mode & kModeNoOut)) {
    // kept values leave through TMA stores of 128 x 32 tiles
    if (!encode_bf16_2d(&p.tm_vals, vals, K / 2, M, K, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return LYNX_ERR_CUDA;
  }
  p.vals = vals;
  p.meta = static_cast<uint8_t*>(meta);
  p.row_scale = row_scale;
  p.t_out = t_out;
  p.lpart = lpart;
  p.tpart = tpart;
  p.M = M;
  p.K = K;
  p.r = static_cast<int>((mode & kModeLora) ? r : 0);
  p.mode = mode;
  p.split = choose_sparsify_split(M, K, ds->sms);
  p.boxes_per_cta = static_cast<int>(K / 64 / p.split);
  p.kblocks = static_cast<int>((K + 127) / 128);
  p.stall_test = g_stall.load();
  p.skip_finalize = fin != nullptr ? 1 : 0;
  if (fin != nullptr) {
    p.fin_flags = fin->flags;
    p.fin_nflags = static_cast<int>(fin_slices(M));
  }
  p.status = stream_status(ds, stream);
  return map_cuda(launch_sparsify(p, stream));
}

// CTA pairs (256 x 256 tiles) unless the problem is too small to feed them; the
// pair kernel steps K by 128 on both paths
bool use_pair_kernel(int64_t M, int64_t N, int64_t K) {
  return M > 128 && N >= 256 && K % 128 == 0;
}

// fused_x: a_src is the dense X and the pair kernel compresses it itself (the
// shape must take the pair kernel; no metadata is read)
lynx_status run_gemm(DeviceState* ds, const void* a_src, bool sparse, const void* meta,
                     const float* row_scale, const void* T, const void* W, const void* bias,
                     const void* B, int64_t M, int64_t N, int64_t K, int64_t r, void* Y,
                     cudaStream_t stream, const FusedFinalize* fin = nullptr, int act = kActNone,
                     bool fused_x = false) {
  GemmLaunch p;
  std::memset(&p, 0, sizeof(p));
  const bool pair = use_pair_kernel(M, N, K);
  if (fused_x && !pair) return LYNX_ERR_UNSUPPORTED_SHAPE;
  const int bn = pair ? 256 : gemm_bn(N);
  const uint32_t b_rows = pair ? 128u : static_cast<uint32_t>(bn);  // W rows one CTA loads
  if (fused_x) {
    // the dense X in 128 x 64 boxes, as on the dense path
    if (!encode_bf16_2d(&p.tm_a, a_src, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return LYNX_ERR_CUDA;
  } else if (sparse) {
    // pair kernel: 128-byte rows of 64 kept values; single-CTA kernel: 64-byte rows
    if (!encode_bf16_2d(&p.tm_a, a_src, K / 2, M, K, pair ? 64 : 32, 128,
                        pair ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return LYNX_ERR_CUDA;
    // metadata blocks of 2 KB seen as 8 rows of 256 bytes
    if (pair && !encode_u8_2d(&p.tm_e, meta, 256,
                              static_cast<uint64_t>(meta_row_blocks(M)) * ((K + 127) / 128) * 8, 256,
                              256, 8))
      return LYNX_ERR_CUDA;
  } else {
    if (!encode_bf16_2d(&p.tm_a, a_src, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return LYNX_ERR_CUDA;
  }
  if (!encode_bf16_2d(&p.tm_b, W, K, N, K * 2, 64, b_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return LYNX_ERR_CUDA;
  const bool lora = (T != nullptr && B != nullptr);
  if (lora) {
    // boxes of 32 columns; for r % 32 == 16 the last box reads past r, which
    // the TMA fills with zeros (and the kernels skip that half's MMA)
    if (!encode_bf16_2d(&p.tm_t, T, r, M, r * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return LYNX_ERR_CUDA;
    if (!encode_bf16_2d(&p.tm_lb, B, r, N, r * 2, 32, b_rows, CU_TENSOR_MAP_SWIZZLE_64B))
      return LYNX_ERR_CUDA;
  }
  if (pair && !encode_bf16_2d(&p.tm_y, Y, N, M, N * 2, 16, 32, CU_TENSOR_MAP_SWIZZLE_32B))
    return LYNX_ERR_CUDA;
  p.meta = static_cast<const uint8_t*>(meta);
  p.row_scale = row_scale;
  p.bias = bias;
  p.y = Y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = lora ? static_cast<int>(r) : 0;
  p.sparse = sparse ? 1 : 0;
  p.lora = lora ? 1 : 0;
  p.bn = bn;
  p.stall_test = g_stall.load();
  p.act = act;
  p.fused = fused_x ? 1 : 0;
  p.status = stream_status(ds, stream);
  if (pair) {
    const int64_t ntm2 = (M + 255) / 256;
    const int64_t tiles = ntm2 * ((N + 255) / 256);
    // one CTA pair per TPC, no more pairs than the device can hold at once
    int64_t pairs = ds->sms / 2;
    const int fit = gemm_pair_max_clusters(sparse, act, fused_x);
    if (fit > 0 && fit < pairs) pairs = fit;
    p.grid = static_cast<int>(2 * (tiles < pairs ? tiles : pairs));
    // raster group: as many 256-row pair-rows of A as fit in ~64 MB of L2, so
    // the group's A stays resident while W streams once per group (all 18
    // pair-rows of a 4608 x 12288 compressed A: 57 MB)
    const int64_t a_row_bytes = 256 * (sparse ? K : 2 * K);
    int64_t gm = (64ll << 20) / (a_row_bytes > 0 ? a_row_bytes : 1);
    gm = gm < 1 ? 1 : (gm > ntm2 ? ntm2 : gm);
    p.group_m = static_cast<int>(gm);
    if (fin != nullptr && fin->mode != 0) {
      p.fin_mode = fin->mode;
      p.fin_split = fin->split;
      p.fin_lpart = fin->lpart;
      p.fin_tpart = fin->tpart;
      p.fin_scale = fin->scale;
      p.fin_t = fin->t;
      p.fin_flags = fin->flags;
    }
    return map_cuda(launch_gemm_pair(p, stream));
  }
  const int64_t tiles = ((M + 127) / 128) * ((N + bn - 1) / bn);
  p.grid = static_cast<int>(tiles < ds->sms ? tiles : ds->sms);
  p.group_m = 16;
  return map_cuda(launch_gemm(p, stream));
}

}  // namespace

bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, resolve_encode);
  if (g_encode == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, resolve_encode);
  if (g_encode == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sm_count() {
  DeviceState* d = device_state();
  return d ? d->sms : 0;
}

}  // namespace lynx

using namespace lynx;

extern "C" {

const char* lynx_status_string(int status) {
  switch (status) {
    case LYNX_OK: return "LYNX_OK";
    case LYNX_ERR_INVALID_ARG: return "LYNX_ERR_INVALID_ARG";
    case LYNX_ERR_UNSUPPORTED_SHAPE: return "LYNX_ERR_UNSUPPORTED_SHAPE";
    case LYNX_ERR_MISALIGNED: return "LYNX_ERR_MISALIGNED";
    case LYNX_ERR_WORKSPACE_TOO_SMALL: return "LYNX_ERR_WORKSPACE_TOO_SMALL";
    case LYNX_ERR_CUDA: return "LYNX_ERR_CUDA";
    case LYNX_ERR_DEVICE_TIMEOUT: return "LYNX_ERR_DEVICE_TIMEOUT";
    default: return "LYNX_ERR_UNKNOWN";
  }
}

int lynx_version(void) { return (1 << 16) | 0; }

int lynx_lora_rank(void) { return kLoraRankDefault; }

int lynx_lora_rank_supported(int64_t r) { return rank_supported(r) ? 1 : 0; }

size_t lynx_vals_bytes(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return 0;
  return static_cast<size_t>(M) * static_cast<size_t>(K);
}

size_t lynx_meta_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return static_cast<size_t>(meta_row_blocks(M)) * static_cast<size_t>((K + 127) / 128) *
         static_cast<size_t>(kMetaBlockBytes);
}

size_t lynx_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r) {
  (void)N;
  if (M <= 0 || K <= 0) return 0;
  return workspace_layout(M, K, r).total;
}

size_t lynx_sparsify_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return sparsify_workspace(M).total;
}

int lynx_sparsify(const void* X, int64_t M, int64_t K, void* vals, void* meta, float* row_scale,
                  void* workspace, size_t workspace_bytes, void* stream) {
  if (X == nullptr || vals == nullptr || meta == nullptr || workspace == nullptr)
    return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_shape(M, 0, K);
  if (st != LYNX_OK) return st;
  if (!aligned16(X) || !aligned16(vals) || !aligned16(meta) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(row_scale) & 3u) != 0)
    return LYNX_ERR_MISALIGNED;
  const SparsifyWorkspace wl = sparsify_workspace(M);
  if (workspace_bytes < wl.total) return LYNX_ERR_WORKSPACE_TOO_SMALL;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scale = row_scale ? row_scale : reinterpret_cast<float*>(ws + wl.scale);
  return run_sparsify(ds, X, nullptr, M, K, 0, vals, meta, scale, nullptr,
                      reinterpret_cast<float2*>(ws + wl.lpart), nullptr, kModeSelect | kModeScaled,
                      static_cast<cudaStream_t>(stream));
}

int64_t lynx_sparsify_noalloc_max_rows(void) { return LYNX_SPARSIFY_NOALLOC_MAX_ROWS; }

int lynx_sparsify_noalloc(const void* X, int64_t M, int64_t K, void* vals, void* meta,
                          float* row_scale, void* stream) {
  static_assert(kMaxSplit == 8, "noalloc scratch is sized for 8 K-splits");
  if (X == nullptr || vals == nullptr || meta == nullptr) return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_shape(M, 0, K);
  if (st != LYNX_OK) return st;
  if (M > LYNX_SPARSIFY_NOALLOC_MAX_ROWS) return LYNX_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(X) || !aligned16(vals) || !aligned16(meta) ||
      (reinterpret_cast<uintptr_t>(row_scale) & 3u) != 0)
    return LYNX_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  uint8_t* scratch = noalloc_scratch();
  if (scratch == nullptr) return LYNX_ERR_CUDA;
  float* scale = row_scale ? row_scale : reinterpret_cast<float*>(scratch + kNoAllocLpartBytes);
  return run_sparsify(ds, X, nullptr, M, K, 0, vals, meta, scale, nullptr,
                      reinterpret_cast<float2*>(scratch), nullptr, kModeSelect | kModeScaled,
                      static_cast<cudaStream_t>(stream));
}

int lynx_linear(const void* X, const void* W, const void* bias, const void* A, const void* B,
                int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, void* Y,
                void* workspace, size_t workspace_bytes, void* stream) {
  return lynx_linear_act(X, W, bias, A, B, M, N, K, r, skip_sparsify, LYNX_ACT_NONE, Y, workspace,
                         workspace_bytes, stream);
}

}  // extern "C"

namespace {

// The layer's two halves on `stream`: begin = the sparsify pass (or, on the
// dense path with LoRA, the LoRA-down pass) into the workspace; finish = the
// GEMM from it.  reset_flags: finish alone on a workspace an earlier call
// filled (profiling), which first clears the combining step's state words.
lynx_status linear_enqueue(const void* X, const void* W, const void* bias, const void* A, const void* B,
                           int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, int act, void* Y,
                           void* workspace, size_t workspace_bytes, cudaStream_t s, bool do_begin,
                           bool do_finish, bool reset_flags) {
  if (X == nullptr || W == nullptr || Y == nullptr) return LYNX_ERR_INVALID_ARG;
  if (act != LYNX_ACT_NONE && act != LYNX_ACT_GELU_TANH) return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_lora(A, B, r);
  if (st != LYNX_OK) return st;
  st = check_shape(M, N, K);
  if (st != LYNX_OK) return st;
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (A && !aligned16(A)) || (B && !aligned16(B)) || (workspace && !aligned16(workspace)))
    return LYNX_ERR_MISALIGNED;
  const bool lora = A != nullptr;
  const bool need_ws = lora || !skip_sparsify;
  const WorkspaceLayout wl = workspace_layout(M, K, r);
  if (need_ws && (workspace == nullptr || workspace_bytes < wl.total))
    return workspace == nullptr ? LYNX_ERR_INVALID_ARG : LYNX_ERR_WORKSPACE_TOO_SMALL;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* t_buf = lora ? ws + wl.t : nullptr;
  // with the CTA-pair GEMM, the GEMM itself combines the pass's K-range partials
  const bool fused = use_pair_kernel(M, N, K) && (!skip_sparsify || lora);
  FusedFinalize fin;
  if (fused) {
    fin.mode = skip_sparsify ? 2 : 1;
    fin.split = choose_sparsify_split(M, K, ds->sms);
    fin.lpart = reinterpret_cast<const float2*>(ws + wl.lpart);
    fin.tpart = reinterpret_cast<const float*>(ws + wl.tpart);
    fin.scale = reinterpret_cast<float*>(ws + wl.scale);
    fin.t = t_buf;
    fin.flags = reinterpret_cast<uint32_t*>(ws + wl.flags);
  }
  if (do_begin) {
    if (!skip_sparsify) {
      st = run_sparsify(ds, X, A, M, K, r, ws + wl.vals, ws + wl.meta, reinterpret_cast<float*>(ws + wl.scale),
                        t_buf, reinterpret_cast<float2*>(ws + wl.lpart), reinterpret_cast<float*>(ws + wl.tpart),
                        kModeSelect | (lora ? kModeLora : 0), s, fused ? &fin : nullptr);
    } else if (lora) {
      st = run_sparsify(ds, X, A, M, K, r, nullptr, nullptr, nullptr, t_buf, nullptr,
                        reinterpret_cast<float*>(ws + wl.tpart), kModeLora, s, fused ? &fin : nullptr);
    }
    if (st != LYNX_OK) return st;
  }
  if (!do_finish) return LYNX_OK;
  if (reset_flags && fused && cudaMemsetAsync(fin.flags, 0, fin_slices(M) * 4, s) != cudaSuccess)
    return LYNX_ERR_CUDA;
  if (void* ev = g_split_event.load())
    if (cudaEventRecord(static_cast<cudaEvent_t>(ev), s) != cudaSuccess) return LYNX_ERR_CUDA;
  if (!skip_sparsify)
    return run_gemm(ds, ws + wl.vals, true, ws + wl.meta, reinterpret_cast<const float*>(ws + wl.scale),
                    t_buf, W, bias, B, M, N, K, r, Y, s, fused ? &fin : nullptr, act);
  return run_gemm(ds, X, false, nullptr, nullptr, t_buf, W, bias, B, M, N, K, r, Y, s,
                  fused ? &fin : nullptr, act);
}

}  // namespace

extern "C" {

int lynx_linear_act(const void* X, const void* W, const void* bias, const void* A, const void* B,
                    int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, int act, void* Y,
                    void* workspace, size_t workspace_bytes, void* stream) {
  const int part = g_profile_part.load();
  return linear_enqueue(X, W, bias, A, B, M, N, K, r, skip_sparsify, act, Y, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), part != 2, part != 1, part == 2);
}

int lynx_linear_begin(const void* X, const void* W, const void* bias, const void* A, const void* B,
                      int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, int act, void* Y,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return linear_enqueue(X, W, bias, A, B, M, N, K, r, skip_sparsify, act, Y, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), true, false, false);
}

int lynx_linear_finish(const void* X, const void* W, const void* bias, const void* A, const void* B,
                       int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, int act, void* Y,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return linear_enqueue(X, W, bias, A, B, M, N, K, r, skip_sparsify, act, Y, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), false, true, false);
}

int lynx_linear_fused(const void* X, const void* W, const void* bias, const void* A, const void* B,
                      int64_t M, int64_t N, int64_t K, int64_t r, int act, void* Y, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (X == nullptr || W == nullptr || Y == nullptr) return LYNX_ERR_INVALID_ARG;
  if (act != LYNX_ACT_NONE && act != LYNX_ACT_GELU_TANH) return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_lora(A, B, r);
  if (st != LYNX_OK) return st;
  st = check_shape(M, N, K);
  if (st != LYNX_OK) return st;
  // shapes the CTA-pair kernel does not take run the two-pass layer
  if (!use_pair_kernel(M, N, K))
    return lynx_linear_act(X, W, bias, A, B, M, N, K, r, 0, act, Y, workspace, workspace_bytes, stream);
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (A && !aligned16(A)) || (B && !aligned16(B)) || (workspace && !aligned16(workspace)))
    return LYNX_ERR_MISALIGNED;
  const WorkspaceLayout wl = workspace_layout(M, K, r);
  if (workspace == nullptr) return LYNX_ERR_INVALID_ARG;
  if (workspace_bytes < wl.total) return LYNX_ERR_WORKSPACE_TOO_SMALL;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool lora = A != nullptr;
  void* t_buf = lora ? ws + wl.t : nullptr;
  FusedFinalize fin;
  fin.mode = 1;
  fin.split = choose_sparsify_split(M, K, ds->sms);
  fin.lpart = reinterpret_cast<const float2*>(ws + wl.lpart);
  fin.tpart = reinterpret_cast<const float*>(ws + wl.tpart);
  fin.scale = reinterpret_cast<float*>(ws + wl.scale);
  fin.t = t_buf;
  fin.flags = reinterpret_cast<uint32_t*>(ws + wl.flags);
  // the slim pass: the row sums (the selection decides the kept sum) and
  // T = X A^T, no values or metadata
  st = run_sparsify(ds, X, A, M, K, r, nullptr, nullptr, reinterpret_cast<float*>(ws + wl.scale), t_buf,
                    reinterpret_cast<float2*>(ws + wl.lpart), reinterpret_cast<float*>(ws + wl.tpart),
                    kModeSelect | kModeNoOut | (lora ? kModeLora : 0), s, &fin);
  if (st != LYNX_OK) return st;
  if (void* ev = g_split_event.load())
    if (cudaEventRecord(static_cast<cudaEvent_t>(ev), s) != cudaSuccess) return LYNX_ERR_CUDA;
  return run_gemm(ds, X, true, nullptr, nullptr, t_buf, W, bias, B, M, N, K, r, Y, s, &fin, act, true);
}

size_t lynx_linear_host_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const size_t x = align256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
  const size_t y = align256(static_cast<size_t>(M) * static_cast<size_t>(N) * 2);
  return x + y + lynx_workspace_bytes(host_chunk_rows(M), N, K, r);
}

int lynx_linear_host(const void* X_host, const void* W, const void* bias, const void* A, const void* B,
                     int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, void* Y_host,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return lynx_linear_host_act(X_host, W, bias, A, B, M, N, K, r, skip_sparsify, LYNX_ACT_NONE, Y_host,
                              workspace, workspace_bytes, stream);
}

int lynx_linear_host_act(const void* X_host, const void* W, const void* bias, const void* A,
                         const void* B, int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify,
                         int act, void* Y_host, void* workspace, size_t workspace_bytes, void* stream) {
  if (X_host == nullptr || W == nullptr || Y_host == nullptr || workspace == nullptr)
    return LYNX_ERR_INVALID_ARG;
  if (act != LYNX_ACT_NONE && act != LYNX_ACT_GELU_TANH) return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_lora(A, B, r);
  if (st != LYNX_OK) return st;
  st = check_shape(M, N, K);
  if (st != LYNX_OK) return st;
  if (!aligned16(workspace)) return LYNX_ERR_MISALIGNED;
  if (workspace_bytes < lynx_linear_host_workspace_bytes(M, N, K, r)) return LYNX_ERR_WORKSPACE_TOO_SMALL;
  HostPipe* hp = host_pipe();
  if (hp == nullptr) return LYNX_ERR_CUDA;
  std::lock_guard<std::mutex> guard(hp->enqueue);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* x_dev = ws;
  uint8_t* y_dev = ws + align256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
  uint8_t* layer_ws = y_dev + align256(static_cast<size_t>(M) * static_cast<size_t>(N) * 2);
  const int64_t rows = host_chunk_rows(M);
  const size_t layer_bytes = lynx_workspace_bytes(rows, N, K, r);
  const size_t xrow = static_cast<size_t>(K) * 2, yrow = static_cast<size_t>(N) * 2;
  // the copies start after the work already on the caller's stream (which may
  // still use the workspace)
  if (cudaEventRecord(hp->start, s) != cudaSuccess || cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return LYNX_ERR_CUDA;
  int chunk = 0;
  for (int64_t m0 = 0; m0 < M; m0 += rows, ++chunk) {
    const int64_t mc = (M - m0 < rows) ? (M - m0) : rows;
    const size_t off_x = static_cast<size_t>(m0) * xrow, off_y = static_cast<size_t>(m0) * yrow;
    if (cudaMemcpyAsync(x_dev + off_x, static_cast<const uint8_t*>(X_host) + off_x,
                        static_cast<size_t>(mc) * xrow, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
        cudaEventRecord(hp->in_done[chunk], hp->in) != cudaSuccess ||
        cudaStreamWaitEvent(s, hp->in_done[chunk], 0) != cudaSuccess)
      return LYNX_ERR_CUDA;
    st = static_cast<lynx_status>(lynx_linear_act(x_dev + off_x, W, bias, A, B, mc, N, K, r, skip_sparsify,
                                                  act, y_dev + off_y, layer_ws, layer_bytes, s));
    if (st != LYNX_OK) return st;
    if (cudaEventRecord(hp->comp_done[chunk], s) != cudaSuccess ||
        cudaStreamWaitEvent(hp->out, hp->comp_done[chunk], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(Y_host) + off_y, y_dev + off_y, static_cast<size_t>(mc) * yrow,
                        cudaMemcpyDeviceToHost, hp->out) != cudaSuccess)
      return LYNX_ERR_CUDA;
  }
  // later work on the caller's stream (and a synchronize of it) sees Y in host memory
  if (cudaEventRecord(hp->out_done, hp->out) != cudaSuccess || cudaStreamWaitEvent(s, hp->out_done, 0) != cudaSuccess)
    return LYNX_ERR_CUDA;
  return LYNX_OK;
}

int lynx_linear_dense(const void* X, const void* W, const void* bias, const void* A,
                      const void* B, int64_t M, int64_t N, int64_t K, int64_t r, void* Y,
                      void* workspace, size_t workspace_bytes, void* stream) {
  return lynx_linear(X, W, bias, A, B, M, N, K, r, 1, Y, workspace, workspace_bytes, stream);
}

int lynx_sparse_gemm(const void* vals, const void* meta, const void* T, const void* W,
                     const void* bias, const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                     void* Y, void* stream) {
  if (vals == nullptr || meta == nullptr || W == nullptr || Y == nullptr) return LYNX_ERR_INVALID_ARG;
  lynx_status st = check_lora(T, B, r);
  if (st != LYNX_OK) return st;
  st = check_shape(M, N, K);
  if (st != LYNX_OK) return st;
  if (!aligned16(vals) || !aligned16(meta) || !aligned16(W) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (T && !aligned16(T)) || (B && !aligned16(B)))
    return LYNX_ERR_MISALIGNED;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  return run_gemm(ds, vals, true, meta, nullptr, T, W, bias, B, M, N, K, r, Y,
                  static_cast<cudaStream_t>(stream));
}

int lynx_check_error(void* stream, uint32_t* device_code) {
  if (device_code) *device_code = 0;
  DeviceState* ds = device_state();
  if (ds == nullptr) return LYNX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LYNX_ERR_CUDA;
  const int slot = find_stream_slot(ds, s);
  if (slot < 0) return LYNX_OK;  // nothing of this library was launched on the stream
  uint32_t* word = ds->status + slot;
  uint32_t code = 0;
  e = cudaMemcpyAsync(&code, word, sizeof(code), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LYNX_ERR_CUDA;
  if (code != 0) {
    e = cudaMemsetAsync(word, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return LYNX_ERR_CUDA;
  }
  if (device_code) *device_code = code;
  return code != 0 ? LYNX_ERR_DEVICE_TIMEOUT : LYNX_OK;
}

// hardware position of (row m, dense column k) inside the metadata buffer:
// byte offset and the shift of the group's nibble inside that byte
static inline void meta_hw_position(int64_t m, int64_t k, int64_t kblocks, size_t* byte,
                                    int* shift) {
  const int64_t mb = m / 128, kb = k / 128;
  const int64_t mi = m % 128, ki = k % 128;
  const int64_t lane = (mi % 8) + 8 * ((ki / 16) % 2) + 16 * (mi / 16);
  const int64_t word = ki / 32;
  const int64_t bit = (ki % 16) + 16 * ((mi / 8) % 2);
  *byte = static_cast<size_t>((mb * kblocks + kb) * 2048 + lane * 16 + word * 4 + bit / 8);
  *shift = static_cast<int>(bit % 8);
}

int lynx_meta_hw_to_canonical(const uint8_t* hw, uint8_t* canonical, int64_t M, int64_t K) {
  if (hw == nullptr || canonical == nullptr) return LYNX_ERR_INVALID_ARG;
  if (M < 1 || K < 8 || K % 8 != 0) return LYNX_ERR_UNSUPPORTED_SHAPE;
  const int64_t kblocks = (K + 127) / 128;
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t g = 0; g < K / 4; ++g) {
      size_t byte;
      int shift;
      meta_hw_position(m, 4 * g, kblocks, &byte, &shift);
      const uint8_t nib = static_cast<uint8_t>((hw[byte] >> shift) & 0xF);
      uint8_t& dst = canonical[m * (K / 8) + g / 2];
      if (g % 2 == 0)
        dst = nib;
      else
        dst = static_cast<uint8_t>(dst | (nib << 4));
    }
  }
  return LYNX_OK;
}

int lynx_meta_canonical_to_hw(const uint8_t* canonical, uint8_t* hw, int64_t M, int64_t K) {
  if (hw == nullptr || canonical == nullptr) return LYNX_ERR_INVALID_ARG;
  if (M < 1 || K < 8 || K % 8 != 0) return LYNX_ERR_UNSUPPORTED_SHAPE;
  const int64_t kblocks = (K + 127) / 128;
  const int64_t mpad = meta_row_blocks(M) * 128;
  std::memset(hw, 0, lynx_meta_bytes(M, K));
  for (int64_t m = 0; m < mpad; ++m) {
    for (int64_t g = 0; g < K / 4; ++g) {
      uint8_t nib = 0x4;  // positions 0,1: the pattern of an all-zero group
      if (m < M) {
        const uint8_t b = canonical[m * (K / 8) + g / 2];
        nib = static_cast<uint8_t>((g % 2 == 0) ? (b & 0xF) : (b >> 4));
      }
      size_t byte;
      int shift;
      meta_hw_position(m, 4 * g, kblocks, &byte, &shift);
      hw[byte] = static_cast<uint8_t>(hw[byte] | (nib << shift));
    }
  }
  return LYNX_OK;
}

int lynx_debug_set_stall(int enable) { return g_stall.exchange(enable ? 1 : 0); }

void* lynx_profile_set_split_event(void* event) { return g_split_event.exchange(event); }

int lynx_profile_set_part(int part) {
  if (part < 0 || part > 2) return -1;
  return g_profile_part.exchange(part);
}

}  // extern "C"
