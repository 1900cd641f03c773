// lynx_internal.h -- declarations shared by the library's translation units.
// Not part of the public ABI (that is include/lynx.h).
#pragma once

#include <cstdint>
#include <mutex>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace lynx {

// LoRA rank r: any multiple of kLoraRankAlign in [kLoraRankAlign, kLoraRankMax]
// (the MMA N of the down-projection; 64 on the RT-Lynx pages)
constexpr int kLoraRankDefault = 64;
constexpr int kLoraRankAlign = 16;
constexpr int kLoraRankMax = 256;
constexpr int kRowBlock = 128;      // rows per metadata block / per MMA tile
constexpr int kMetaBlockK = 128;    // dense K per metadata block
constexpr int kMetaBlockBytes = 2048;  // 128 TMEM lanes x 16 bytes

// ---- sparsify / LoRA-down pass ---------------------------------------------

// kModeSelect: S(X) (kept values + metadata + s); kModeLora: T = X A^T;
// kModeScaled: values leave compensated (standalone S(X)), otherwise they
// leave as kept and s is applied by the GEMM (T is then written as T / s);
// kModeNoOut (with kModeSelect): the selection only feeds the row sums, no
// values or metadata are written (the fused GEMM selects again from X).
enum SparsifyMode : int { kModeSelect = 1, kModeLora = 2, kModeScaled = 4, kModeNoOut = 8 };

// Activation the GEMM epilogue applies to each finished output value (the
// LYNX_ACT_* values of the public header).
enum EpilogueAct : int { kActNone = 0, kActGeluTanh = 1 };

constexpr int kMaxSplit = 8;  // K ranges per row block in the sparsify pass

struct SparsifyLaunch {
  CUtensorMap tm_x;     // X [M,K] bf16, box 64 x 128, 128B swizzle
  CUtensorMap tm_a;     // A [r,K] bf16, box 64 x r, 128B swizzle (mode & kModeLora)
  CUtensorMap tm_vals;  // vals [M,K/2] bf16, box 32 x 128, 64B swizzle (stores)
  void* vals;           // [M, K/2] bf16 (mode & kModeSelect)
  uint8_t* meta;        // hardware-layout metadata blocks (mode & kModeSelect)
  float* row_scale;     // [M] s per row (mode & kModeSelect)
  void* t_out;          // [M, r] bf16 (mode & kModeLora)
  float2* lpart;        // [split][M] partial (sum|x|, sum|kept|) per K range
  float* tpart;         // [split][M][r] partial T per K range
  int64_t M, K;
  int r;                // LoRA rank (mode & kModeLora)
  int mode;
  int split;            // K ranges per row block (1..kMaxSplit, divides K/64)
  int boxes_per_cta;    // 64-column boxes each CTA covers
  int kblocks;          // metadata blocks per row block: ceil(K/128)
  int stall_test;       // test-only: the producer never loads, waits must time out
  int skip_finalize;    // the GEMM that follows combines the partials (finalize_kernel not launched)
  // With skip_finalize: the GEMM's per-slice state words, set to 0 by the
  // pass's first CTA (the GEMM claims and publishes each 32-row slice of the
  // partials' combination through them)
  uint32_t* fin_flags;
  int fin_nflags;
  uint32_t* status;     // the stream's status word (first error code wins)
};

// sparsify pass + finalize (+ rescale for the standalone form), on one stream
// Launches `kernel` with programmatic stream serialization: it may begin (and
// run its prologue) while the previous kernel on `stream` finishes; it must call
// pdl_wait() before it reads anything that kernel wrote.
template <typename... Params, typename... Args>
cudaError_t launch_after_previous(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_sparsify(const SparsifyLaunch& p, cudaStream_t stream);
int choose_sparsify_split(int64_t M, int64_t K, int num_sms);
size_t sparsify_smem_bytes(int mode, int r);

// ---- tcgen05 GEMM with LoRA-up + bias epilogue ------------------------------

struct GemmLaunch {
  CUtensorMap tm_a;     // sparse: vals [M,K/2] box 32x128 SW64; dense: X [M,K] box 64x128 SW128
  CUtensorMap tm_b;     // W [N,K] box 64 x BN, SW128
  CUtensorMap tm_t;     // T [M,r] box 32 x 128, SW64 (lora)
  CUtensorMap tm_lb;    // B [N,r] box 32 x BN, SW64 (lora)
  CUtensorMap tm_e;     // metadata as uint8 [blocks*8, 256], box 256 x 8 (pair kernel)
  CUtensorMap tm_y;     // Y [M,N] bf16, box 16 x 32, 32B swizzle (pair kernel stores)
  const uint8_t* meta;  // hardware metadata blocks (sparse)
  const void* bias;     // [N] bf16 or null
  const float* row_scale;  // [M] fp32 multiplier of each accumulator row, or null
  void* y;              // [M,N] bf16
  int64_t M, N, K;
  int r;                // LoRA rank (lora)
  int sparse;
  int lora;
  int bn;               // 128 or 256
  int grid;             // persistent CTAs
  int group_m;          // tile rows (of 128 or of 256 for CTA pairs) per raster group
  int stall_test;
  int act;              // EpilogueAct
  int fused;            // pair kernel: A is the dense X, compressed in the kernel (tm_a maps X)
  uint32_t* status;
  // Combining the sparsify pass's K-range partials inside the pair GEMM (instead
  // of finalize_kernel): fin_mode 1 = s (and, with LoRA, bf16(T / s)), 2 =
  // bf16(T) only, 0 = off.  Each 32-row slice has a state word in fin_flags
  // (0 = open, 1 = being combined, 2 = done), which the sparsify pass of the
  // same call sets to 0.  Before its first tile, a CTA's epilogue warps claim
  // (0 -> 1), combine and publish (2) the slices it owns, then check the slices
  // of its tiles, combining any still open and waiting for those another
  // running CTA holds.  The producer loads T after they have seen all done.
  int fin_mode;
  int fin_split;
  const float2* fin_lpart;
  const float* fin_tpart;
  float* fin_scale;
  void* fin_t;
  uint32_t* fin_flags;  // one word per 32-row slice (fin_slices(M))
};

cudaError_t launch_gemm(const GemmLaunch& p, cudaStream_t stream);       // 128 x BN tiles, 1 CTA
cudaError_t launch_gemm_pair(const GemmLaunch& p, cudaStream_t stream);  // 256 x 256 tiles, CTA pairs
// CTA pairs of the pair GEMM (this variant) that the current device can hold at
// once; 0 if the query failed.  Computed once per device and variant.
int gemm_pair_max_clusters(bool sparse, int act, bool fused = false);

// Per-device one-time set-up of a kernel's dynamic shared-memory limit:
// `configure` runs once for each device (thread-safe); its result is kept.
template <typename F>
cudaError_t once_per_device(std::once_flag (&flags)[64], cudaError_t (&results)[64], F&& configure) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(flags[dev], [&]() { results[dev] = configure(); });
  return results[dev];
}

// ---- helpers ----------------------------------------------------------------

// 128-row blocks of metadata are allocated in pairs (a CTA pair covers 256 rows)
inline int64_t meta_row_blocks(int64_t M) { return (M + 255) / 256 * 2; }

// 32-row slices of the pair GEMM's combining step (one state word each)
inline int64_t fin_slices(int64_t M) { return (M + 31) / 32; }

// 2-D uint8 tensor map (no swizzle)
bool encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// 2-D bf16 tensor map: inner (contiguous) extent, outer extent, row pitch in bytes
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);

int device_sm_count();

}  // namespace lynx
