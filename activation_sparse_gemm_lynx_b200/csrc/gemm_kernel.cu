// gemm_kernel.cu -- persistent tcgen05 GEMM for the Lynx layer:
//   Y[M,N] = bf16( S(X) W^T  (+ T B^T)  (+ bias) )
// with S(X) either the 2:4-compressed activations (tcgen05.mma.sp, sparse
// operand on the A side, metadata in TMEM) or the dense X (tcgen05.mma, the
// path of layers left dense by selective layer skipping).  T = X A^T is the
// LoRA down-projection produced by the sparsify pass; the LoRA up-projection
// runs as two extra dense K=32 steps into the same TMEM accumulator tile, and
// the bias is added in fp32 before the single bf16 rounding of Y (after an
// optional activation, GELU tanh form, also in fp32).
// (RT-Lynx pages: qingkeai.online article section 02, Y = S(X) W^T; section
// 03.2, LoRA residual; section 03.3, skipped layers; section 04, sparse GEMM
// and LoRA residual fused into the CUDA kernel.)
//
// Tile: 128 rows x BN columns per CTA, one CTA per SM (persistent, static
// round-robin over tiles, M-grouped raster for L2 reuse).
//   warp 0      TMA producer: A tile (vals 128x32 compressed, 64B swizzle, or
//               X 128x64, 128B swizzle), W tile (BNx64, 128B swizzle) and, every
//               second stage of the sparse path, one 2 KB metadata block (plain
//               bulk copy).  LoRA stages: T (128x32) and B (BNx32), 64B swizzle.
//   warp 1      TMEM owner + MMA issuer (one thread): tcgen05.cp of metadata
//               into a 4-slot TMEM ring, tcgen05.mma(.sp) into the accumulator,
//               tcgen05.commit to release stages / publish the accumulator.
//   warps 2-9   epilogue: tcgen05.ld 32x32b -> s * acc + bias -> bf16 -> global
//               (two warps per TMEM lane quarter, half of the columns each).
// Accumulators: 1 TMEM buffer for BN = 256, 2 (double buffered) for BN = 128.
#include <cuda_bf16.h>

#include "lynx_act.cuh"
#include "lynx_internal.h"
#include "lynx_ptx.cuh"

namespace lynx {

namespace {

constexpr int kGemmThreads = 320;  // producer, MMA, 8 epilogue warps
constexpr uint32_t kTmemCols = 512;
constexpr int kGroupM = 16;
constexpr int kEslots = 4;

template <int BN, bool SPARSE>
struct Cfg {
  static constexpr uint32_t kABytes = SPARSE ? 128u * 64u : 128u * 128u;  // one k-step of A
  static constexpr uint32_t kBBytes = static_cast<uint32_t>(BN) * 128u;   // BN rows x 64 dense K
  static constexpr uint32_t kEBytes = SPARSE ? 2048u : 0u;
  static constexpr uint32_t kStageBytes = ((kABytes + kBBytes + kEBytes + 1023u) / 1024u) * 1024u;
  static constexpr int kStages = static_cast<int>((212u * 1024u) / kStageBytes);
  static constexpr int kAcc = BN > 128 ? 1 : 2;
  static constexpr uint32_t kEcol0 = static_cast<uint32_t>(kAcc * BN);
  static constexpr uint32_t kLoraABytes = 128u * 64u;                     // T: 128 rows x 32
  static constexpr uint32_t kLoraBBytes = static_cast<uint32_t>(BN) * 64u;  // B: BN rows x 32
  static_assert(kStages >= 3, "pipeline too shallow");
  static_assert(kEcol0 + 4 * kEslots <= kTmemCols, "TMEM budget");
};

template <int BN, bool SPARSE>
struct __align__(1024) GemmSmem {
  using C = Cfg<BN, SPARSE>;
  uint8_t stage[C::kStages][C::kStageBytes];
  uint64_t full[C::kStages];
  uint64_t empty[C::kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  float bias_s[BN];  // the current tile's bias, fp32
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

constexpr uint32_t kBarEpilogue = 2;  // named barrier of the 8 epilogue warps
constexpr uint32_t kEpiThreads = 256;

__device__ __forceinline__ void tile_coords(int tile, int ntm, int ntn, int& mb, int& nb) {
  const int per_group = kGroupM * ntn;
  const int group = tile / per_group;
  const int first_m = group * kGroupM;
  const int gm = min(kGroupM, ntm - first_m);
  const int in_group = tile - group * per_group;
  mb = first_m + in_group % gm;
  nb = in_group / gm;
}

template <int BN, bool SPARSE>
__global__ void __launch_bounds__(kGemmThreads, 1)
lynx_gemm_kernel(const __grid_constant__ GemmLaunch p) {
  using C = Cfg<BN, SPARSE>;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem<BN, SPARSE>& sm = *reinterpret_cast<GemmSmem<BN, SPARSE>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int ntm = static_cast<int>((p.M + 127) / 128);
  const int ntn = static_cast<int>((p.N + BN - 1) / BN);
  const int ntiles = ntm * ntn;
  const int nk = static_cast<int>(p.K / 64);  // 64 dense K per stage
  const int kblocks = static_cast<int>((p.K + 127) / 128);
  const bool lora = p.lora != 0;
  const int lsteps = lora ? (p.r + 31) / 32 : 0;  // LoRA-up stages of K = 32 (zero-filled past r)

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 8);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the prologue above may overlap the previous kernel (programmatic launch);
  // its outputs are read only from here on
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_b);
      if (lora) {
        tma_prefetch_desc(&p.tm_t);
        tma_prefetch_desc(&p.tm_lb);
      }
      uint32_t g = 0;
      bool ok = !p.stall_test;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, ntm, ntn, mb, nb);
        const int32_t row0 = mb * 128;
        const int32_t col0 = nb * BN;
        const int steps = nk + lsteps;
        for (int kit = 0; kit < steps; ++kit, ++g) {
          const uint32_t slot = g % C::kStages;
          const uint32_t ph = (g / C::kStages) & 1u;
          if (sm.abort_flag || !mbar_wait(&sm.empty[slot], ph ^ 1u)) {
            if (!sm.abort_flag) {
              record_error(p.status, kDevTimeoutEmpty);
              sm.abort_flag = 1u;
            }
            ok = false;
            break;
          }
          uint8_t* st = sm.stage[slot];
          if (kit < nk) {
            const bool load_e = SPARSE && (kit % 2 == 0);
            mbar_arrive_expect_tx(&sm.full[slot], C::kABytes + C::kBBytes + (load_e ? 2048u : 0u));
            if (SPARSE)
              tma_load_2d(st, &p.tm_a, &sm.full[slot], kit * 32, row0);
            else
              tma_load_2d(st, &p.tm_a, &sm.full[slot], kit * 64, row0);
            tma_load_2d(st + C::kABytes, &p.tm_b, &sm.full[slot], kit * 64, col0);
            if (load_e) {
              const uint8_t* src =
                  p.meta + (static_cast<size_t>(mb) * kblocks + kit / 2) * kMetaBlockBytes;
              bulk_load(st + C::kABytes + C::kBBytes, src, 2048u, &sm.full[slot]);
            }
          } else {
            const int l = kit - nk;
            mbar_arrive_expect_tx(&sm.full[slot], C::kLoraABytes + C::kLoraBBytes);
            tma_load_2d(st, &p.tm_t, &sm.full[slot], l * 32, row0);
            tma_load_2d(st + C::kABytes, &p.tm_lb, &sm.full[slot], l * 32, col0);
          }
        }
      }
      // drain: the last fill of every stage must have landed before exit
      const uint32_t issued = g;
      for (uint32_t b = issued; b > 0 && b + C::kStages > issued; --b) {
        const uint32_t x = b - 1;
        if (!mbar_wait(&sm.full[x % C::kStages], (x / C::kStages) & 1u, kWaitLimitNs / 4))
          record_error(p.status, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_main = make_idesc_bf16(128, BN, SPARSE);
      const uint32_t idesc_dense = make_idesc_bf16(128, BN, false);
      uint32_t g = 0, eslot = 0;
      int acc_count = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++acc_count) {
        const int acc = acc_count % C::kAcc;
        const uint32_t acc_ph = static_cast<uint32_t>(acc_count / C::kAcc) & 1u;
        if (sm.abort_flag || !mbar_wait(&sm.acc_empty[acc], acc_ph ^ 1u)) {
          if (!sm.abort_flag) {
            record_error(p.status, kDevTimeoutAccum);
            sm.abort_flag = 1u;
          }
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = sm.tmem_base + static_cast<uint32_t>(acc * BN);
        const int steps = nk + lsteps;
        uint32_t accumulate = 0;
        for (int kit = 0; kit < steps; ++kit, ++g) {
          const uint32_t slot = g % C::kStages;
          const uint32_t ph = (g / C::kStages) & 1u;
          if (sm.abort_flag || !mbar_wait(&sm.full[slot], ph)) {
            if (!sm.abort_flag) {
              record_error(p.status, kDevTimeoutFull);
              sm.abort_flag = 1u;
            }
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm.stage[slot]);
          const uint32_t sb = sa + C::kABytes;
          if (kit < nk) {
            if (SPARSE) {
              if (kit % 2 == 0) {
                eslot = (eslot + 1) % kEslots;
                const uint64_t edesc = make_sdesc(sb + C::kBBytes, 2048, 128, kSwNone);
                tc_cp_128x128b(sm.tmem_base + C::kEcol0 + 4 * eslot, edesc);
              }
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t ecol = C::kEcol0 + 4 * eslot + 2 * (kit % 2) + j;
                const uint64_t da = make_sdesc(sa + 32 * j, 16, 512, kSw64);
                const uint64_t db = make_sdesc(sb + 64 * j, 16, 1024, kSw128);
                const uint32_t idesc = idesc_main | (ecol & 1u);
                mma_sp_bf16(d_tmem, da, db, sm.tmem_base + (ecol & ~1u), idesc, accumulate);
                accumulate = 1;
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t da = make_sdesc(sa + 32 * kk, 16, 1024, kSw128);
                const uint64_t db = make_sdesc(sb + 32 * kk, 16, 1024, kSw128);
                mma_bf16(d_tmem, da, db, idesc_main, accumulate);
                accumulate = 1;
              }
            }
          } else {
            const int l = kit - nk;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              if (32 * l + 16 * kk >= p.r) break;  // past r: the zero-filled half of the box
              const uint64_t da = make_sdesc(sa + 32 * kk, 16, 512, kSw64);
              const uint64_t db = make_sdesc(sb + 32 * kk, 16, 512, kSw64);
              mma_bf16(d_tmem, da, db, idesc_dense, accumulate);
              accumulate = 1;
            }
          }
          tc_commit(&sm.empty[slot]);
        }
        if (!ok) break;
        tc_commit(&sm.acc_full[acc]);
      }
      tc_commit(&sm.drain);
      if (!mbar_wait(&sm.drain, 0)) record_error(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Y = bf16(act(s_row * acc + bias)).  Two warps per TMEM lane quarter, each
    // draining half of the columns into registers; the TMEM buffer is released
    // before the global stores, so the next tile's MMAs overlap them.
    constexpr int kHalf = BN / 2;
    const uint32_t q = warp & 3u;              // TMEM lane quarter this warp may access
    const uint32_t ch = (warp - 2u) >> 2;      // which half of the columns
    const uint32_t row = 32u * q + lane;
    const uint32_t et = threadIdx.x - 64u;     // 0..255
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.y);
    int acc_count = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++acc_count) {
      int mb, nb;
      tile_coords(tile, ntm, ntn, mb, nb);
      const int acc = acc_count % C::kAcc;
      const uint32_t acc_ph = static_cast<uint32_t>(acc_count / C::kAcc) & 1u;
      const int64_t grow = static_cast<int64_t>(mb) * 128 + row;
      const bool row_ok = grow < p.M;
      const int64_t n_base = static_cast<int64_t>(nb) * BN;
      named_bar_sync(kBarEpilogue, kEpiThreads);  // the previous tile's bias is no longer read
      for (uint32_t j = et; j < static_cast<uint32_t>(BN); j += kEpiThreads) {
        const int64_t n = n_base + j;
        sm.bias_s[j] = (bias != nullptr && n < p.N) ? __bfloat162float(bias[n]) : 0.f;
      }
      const float s = (p.row_scale != nullptr && row_ok) ? p.row_scale[grow] : 1.f;
      bool ok = !sm.abort_flag;
      if (ok && !mbar_wait(&sm.acc_full[acc], acc_ph)) {
        record_error(p.status, kDevTimeoutAccum);
        sm.abort_flag = 1u;
        ok = false;
      }
      // publishes the bias tile and makes the stop decision identical in all warps
      if (named_bar_red_or(kBarEpilogue, kEpiThreads, !ok)) break;
      tc_fence_after();
      uint32_t out[kHalf / 2];
#pragma unroll
      for (int c = 0; c < kHalf / 32; ++c) {
        const int col = static_cast<int>(ch) * kHalf + 32 * c;
        uint32_t r[32];
        tmem_ld_32x32b_x32(sm.tmem_base + ((32u * q) << 16) + static_cast<uint32_t>(acc * BN + col), r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a = __fmaf_rn(s, __uint_as_float(r[2 * i]), sm.bias_s[col + 2 * i]);
          float b = __fmaf_rn(s, __uint_as_float(r[2 * i + 1]), sm.bias_s[col + 2 * i + 1]);
          if (p.act == kActGeluTanh) {
            a = gelu_tanh(a);
            b = gelu_tanh(b);
          }
          __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
          out[16 * c + i] = *reinterpret_cast<uint32_t*>(&h);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
      if (row_ok) {
        const int64_t n0 = n_base + static_cast<int64_t>(ch) * kHalf;
        __nv_bfloat16* yrow = y + grow * p.N + n0;
#pragma unroll
        for (int v = 0; v < kHalf / 8; ++v) {
          if (n0 + 8 * v < p.N)
            *reinterpret_cast<uint4*>(yrow + 8 * v) =
                make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2], out[4 * v + 3]);
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) tmem_dealloc(sm.tmem_base, kTmemCols);
}

template <int BN, bool SPARSE>
cudaError_t launch_variant(const GemmLaunch& p, cudaStream_t stream) {
  const size_t smem = sizeof(GemmSmem<BN, SPARSE>) + 1024;
  static std::once_flag once[64];
  static cudaError_t configured[64];
  cudaError_t e = once_per_device(once, configured, [smem]() {
    return cudaFuncSetAttribute(lynx_gemm_kernel<BN, SPARSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
  });
  if (e != cudaSuccess) return e;
  return launch_after_previous(lynx_gemm_kernel<BN, SPARSE>, dim3(static_cast<unsigned>(p.grid)),
                               dim3(kGemmThreads), smem, stream, p);
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& p, cudaStream_t stream) {
  if (p.bn == 256)
    return p.sparse ? launch_variant<256, true>(p, stream) : launch_variant<256, false>(p, stream);
  return p.sparse ? launch_variant<128, true>(p, stream) : launch_variant<128, false>(p, stream);
}

}  // namespace lynx
