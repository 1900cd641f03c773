// sparsify_kernel.cu -- online 2:4 activation sparsification with norm
// compensation, plus the LoRA down-projection T = X A^T from the same read of X.
//
// What it computes (RT-Lynx pages: qingkeai.online article sections 02-04;
// ai-feeds.com summary "core module 1"):
//   per token row m and group g of 4 consecutive K values: keep the 2 largest
//   magnitudes (ties to the lower index); L_all = sum|x|, L_kept = sum|kept|
//   (fp32); s = L_all / L_kept (1 if L_kept == 0); kept values v' = bf16(v*s),
//   stored compressed (2 per group, ascending position) together with the
//   2-bit positions in the operand layout of tcgen05.mma.sp; optionally
//   T = X A^T (fp32 accumulate on tensor cores, stored as bf16).
//
// Organisation (one launch):
//   grid = (C, ceil(M/128)), cluster = (C,1,1): the C CTAs of a cluster share
//   one 128-row block and split K into C equal ranges.
//   warp 0      TMA producer: 128x64 tiles of X (and 64x64 tiles of A) into a
//               3-stage ring (128-byte swizzle, the UMMA K-major layout)
//   warp 1      owns TMEM (64 columns) and issues tcgen05.mma M=128,N=64,K=16
//               on each X tile for the LoRA down-projection
//   warps 2..9  256 "row threads": thread = (row, half of each 64-wide tile).
//               Selection, fp32 partial sums, unscaled kept values and
//               metadata go out as the tiles stream by.
//   After the ring: partial sums of the C CTAs are combined in a fixed order
//   over distributed shared memory (deterministic), every CTA derives s, the
//   T partials are reduced column-slice-wise the same way, and a second sweep
//   rescales the kept values this thread wrote moments ago (an L2 hit).
//
// Metadata layout (what tcgen05.cp.128x128b + tcgen05.mma.sp kind::f16 with
// M=128 consume): one 2048-byte block per 128 rows x 128 dense K, stored as
// 128 TMEM lanes x 16 bytes.  For row m (within the block) and dense column k
// (within the block): lane = (m & 7) + 8*((k >> 4) & 1) + 16*(m >> 4), 32-bit
// word = k >> 5, bit = (k & 15) + 16*((m >> 3) & 1) with 4 bits per group:
// the group's nibble lo | hi << 2.  Blocks are ordered row-block major:
// block (mb, kb) starts at byte (mb * ceil(K/128) + kb) * 2048.
#include <cuda_bf16.h>

#include "lynx_internal.h"
#include "lynx_ptx.cuh"

namespace lynx {

namespace {

constexpr int kStages = 3;
constexpr int kComputeWarps = 8;
constexpr int kThreads = 64 + 32 * kComputeWarps;  // 320
constexpr uint32_t kXTileBytes = 128 * 64 * 2;       // 16 KB
constexpr uint32_t kATileBytes = 64 * 64 * 2;        // 8 KB
constexpr uint32_t kTmemCols = 64;

struct __align__(1024) SparsifySmem {
  uint8_t xring[kStages][kXTileBytes];
  uint8_t aring[kStages][kATileBytes];
  float recv[128 * 64];          // T partial slices from every CTA of the cluster
  float2 part[128];              // this CTA's (L_all, L_kept) per row
  float2 halfpart[128];          // second half-tile partials, combined locally
  float srow[128];               // final s per row
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tdone;
  uint64_t drain;
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

__device__ __forceinline__ float abs_lo(uint32_t w) { return __uint_as_float((w << 16) & 0x7FFFFFFFu); }
__device__ __forceinline__ float abs_hi(uint32_t w) { return __uint_as_float(w & 0x7FFF0000u); }

// Top-2 of the 4 bf16 values in (w0 = x1:x0, w1 = x3:x2) by magnitude, ties to
// the lower index.  Each value becomes a distinct key (|x| << 2) | (3 - i), so
// a larger key is a larger magnitude or, on equal magnitude, a lower index.
// Returns the nibble lo | hi << 2 and the kept pair packed (x_lo in the low
// half), and adds the group's magnitudes to the running fp32 sums in k order.
__device__ __forceinline__ uint32_t select_group(uint32_t w0, uint32_t w1, uint32_t& kept,
                                                 float& l_all, float& l_kept) {
  const uint32_t k0 = ((w0 << 2) & 0x1FFFCu) | 3u;
  const uint32_t k1 = ((w0 >> 14) & 0x1FFFCu) | 2u;
  const uint32_t k2 = ((w1 << 2) & 0x1FFFCu) | 1u;
  const uint32_t k3 = ((w1 >> 14) & 0x1FFFCu);
  const uint32_t p = max(k0, k1), q = min(k0, k1);
  const uint32_t r = max(k2, k3), u = min(k2, k3);
  const uint32_t t1 = max(p, r);
  const uint32_t t2 = max(min(p, r), max(q, u));
  const uint32_t a = t1 & 3u, b = t2 & 3u;  // 3 - index of the two winners
  const uint32_t lo = 3u - max(a, b);
  const uint32_t hi = 3u - min(a, b);
  // byte selector picking elements lo and hi out of the 8 bytes (w1:w0)
  const uint32_t sel = 0x1010u + lo * 0x22u + hi * 0x2200u;
  kept = __byte_perm(w0, w1, sel);
  l_all = __fadd_rn(l_all, abs_lo(w0));
  l_all = __fadd_rn(l_all, abs_hi(w0));
  l_all = __fadd_rn(l_all, abs_lo(w1));
  l_all = __fadd_rn(l_all, abs_hi(w1));
  l_kept = __fadd_rn(l_kept, abs_lo(kept));
  l_kept = __fadd_rn(l_kept, abs_hi(kept));
  return lo | (hi << 2);
}

__device__ __forceinline__ uint32_t scale_pair(uint32_t w, float s) {
  const float a = __fmul_rn(__uint_as_float(w << 16), s);
  const float b = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), s);
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void set_abort(SparsifySmem& sm, uint32_t* status, uint32_t code) {
  record_error(status, code);
  sm.abort_flag = 1u;
}

__global__ void __launch_bounds__(kThreads, 2)
sparsify_kernel(const __grid_constant__ SparsifyLaunch p) {
  extern __shared__ uint8_t smem_raw[];
  SparsifySmem& sm = *reinterpret_cast<SparsifySmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();   // == blockIdx.x
  const uint32_t C = static_cast<uint32_t>(p.cluster);
  const int64_t mb = blockIdx.y;
  const int nboxes = p.boxes_per_cta;
  const bool do_sel = (p.mode & kModeSelect) != 0;
  const bool do_lora = (p.mode & kModeLora) != 0;
  const int64_t kcol0 = static_cast<int64_t>(rank) * nboxes * 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], (do_sel ? kComputeWarps : 0) + (do_lora ? 1 : 0));
    }
    mbar_init(&sm.tdone, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 1 && do_lora) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_x);
      if (do_lora) tma_prefetch_desc(&p.tm_a);
      const uint32_t tx = kXTileBytes + (do_lora ? kATileBytes : 0u);
      int issued = 0;
      if (!p.stall_test) {
        for (int b = 0; b < nboxes; ++b) {
          const int slot = b % kStages;
          const uint32_t it = static_cast<uint32_t>(b / kStages);
          if (sm.abort_flag) break;
          if (!mbar_wait(&sm.empty[slot], (it & 1u) ^ 1u)) {
            set_abort(sm, p.status, kDevTimeoutEmpty);
            break;
          }
          mbar_arrive_expect_tx(&sm.full[slot], tx);
          const int32_t kc = static_cast<int32_t>(kcol0 + 64 * b);
          tma_load_2d(sm.xring[slot], &p.tm_x, &sm.full[slot], kc, static_cast<int32_t>(mb * 128));
          if (do_lora) tma_load_2d(sm.aring[slot], &p.tm_a, &sm.full[slot], kc, 0);
          ++issued;
        }
      }
      // never leave with copies in flight: wait for the last fill of each slot
      for (int b = issued - 1; b >= 0 && b >= issued - kStages; --b) {
        if (!mbar_wait(&sm.full[b % kStages], static_cast<uint32_t>(b / kStages) & 1u, kWaitLimitNs / 4))
          record_error(p.status, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ LoRA-down MMA
    if (do_lora && lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, kLoraRank, false);
      const uint32_t t_tmem = sm.tmem_base;
      for (int b = 0; b < nboxes; ++b) {
        const int slot = b % kStages;
        const uint32_t it = static_cast<uint32_t>(b / kStages);
        if (sm.abort_flag) break;
        if (!mbar_wait(&sm.full[slot], it & 1u)) {
          set_abort(sm, p.status, kDevTimeoutFull);
          break;
        }
        tc_fence_after();
        const uint32_t xa = smem_u32(sm.xring[slot]);
        const uint32_t aa = smem_u32(sm.aring[slot]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = make_sdesc(xa + 32 * kk, 16, 1024, kSw128);
          const uint64_t db = make_sdesc(aa + 32 * kk, 16, 1024, kSw128);
          mma_bf16(t_tmem, da, db, idesc, (b | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&sm.empty[slot]);
      }
      tc_commit(&sm.tdone);
      // all MMAs issued so far are complete once this fires (used on every path)
      tc_commit(&sm.drain);
      if (!mbar_wait(&sm.drain, 0)) record_error(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (do_sel) {
    // ------------------------------------------------------------ row threads
    const uint32_t half = (warp - 2) >> 2;
    const uint32_t row = 32 * (warp & 3) + lane;
    const int64_t grow = mb * 128 + row;
    const bool row_ok = grow < p.M;
    const uint32_t meta_lane0 = (row & 7) + 16 * (row >> 4);
    const uint32_t meta_hsel = (row >> 3) & 1;
    uint16_t* meta_blk_base =
        reinterpret_cast<uint16_t*>(p.meta + static_cast<size_t>(mb) * p.kblocks * kMetaBlockBytes);
    uint4* vrow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.vals) +
                                           static_cast<size_t>(grow) * p.K);  // K/2 bf16 = K bytes
    float l_all = 0.f, l_kept = 0.f;
    for (int b = 0; b < nboxes; ++b) {
      const int slot = b % kStages;
      const uint32_t it = static_cast<uint32_t>(b / kStages);
      if (sm.abort_flag) break;
      if (!mbar_wait(&sm.full[slot], it & 1u)) {
        set_abort(sm, p.status, kDevTimeoutFull);
        break;
      }
      const uint8_t* tile = sm.xring[slot];
      uint32_t kw[8];
      uint32_t nib16[2];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t chunk = 4 * half + q;
        const uint4 v = *reinterpret_cast<const uint4*>(tile + row * 128 + ((chunk ^ (row & 7)) << 4));
        const uint32_t n0 = select_group(v.x, v.y, kw[2 * q], l_all, l_kept);
        const uint32_t n1 = select_group(v.z, v.w, kw[2 * q + 1], l_all, l_kept);
        const uint32_t bits8 = n0 | (n1 << 4);
        if (q & 1)
          nib16[q >> 1] |= bits8 << 8;
        else
          nib16[q >> 1] = bits8;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      // metadata: this thread covers dense columns [kabs, kabs+32) of its row
      const int64_t kabs = kcol0 + 64 * b + 32 * half;
      const int64_t kb = kabs >> 7;
      const uint32_t c32 = static_cast<uint32_t>((kabs & 127) >> 5);
      uint16_t* blk = meta_blk_base + static_cast<size_t>(kb) * (kMetaBlockBytes / 2);
      blk[(meta_lane0) * 8 + c32 * 2 + meta_hsel] = static_cast<uint16_t>(nib16[0]);
      blk[(meta_lane0 + 8) * 8 + c32 * 2 + meta_hsel] = static_cast<uint16_t>(nib16[1]);
      if (row_ok) {
        uint4* dst = vrow + (kabs >> 4);  // kabs/2 bf16 = kabs bytes = kabs/16 uint4
        dst[0] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        dst[1] = make_uint4(kw[4], kw[5], kw[6], kw[7]);
      }
    }
    if (half == 1) sm.halfpart[row] = make_float2(l_all, l_kept);
    named_bar_sync(1, 32 * kComputeWarps);
    if (half == 0) {
      const float2 o = sm.halfpart[row];
      sm.part[row] = make_float2(__fadd_rn(l_all, o.x), __fadd_rn(l_kept, o.y));
    }
  }

  // ---- T partial: TMEM -> registers -> owner CTA's receive buffer (by column slice)
  if (do_lora && warp >= 2 && warp < 6) {
    const uint32_t row = 32 * (warp & 3) + lane;
    if (!sm.abort_flag && mbar_wait(&sm.tdone, 0)) {
      tc_fence_after();
      const uint32_t w = kLoraRank / C;  // columns owned by each CTA
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(sm.tmem_base + ((32u * (warp & 3)) << 16) + 32u * h, r);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const uint32_t col = 32 * h + c;
          const uint32_t owner = col / w;
          const uint32_t off = col % w;
          const uint32_t dst = mapa_shared(
              smem_u32(&sm.recv[(rank * 128 + row) * w + off]), owner);
          st_cluster_v4(dst, __uint_as_float(r[c]), __uint_as_float(r[c + 1]),
                        __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
        }
      }
      tc_fence_before();
    } else if (!sm.abort_flag) {
      set_abort(sm, p.status, kDevTimeoutAccum);
    }
  }

  __syncwarp();
  cluster_sync_all();  // partial sums and T slices are published cluster-wide

  if (warp >= 2 && warp < 6) {
    const uint32_t row = 32 * (warp & 3) + lane;
    const int64_t grow = mb * 128 + row;
    if (do_sel) {
      float la = 0.f, lk = 0.f;
      const uint32_t my = smem_u32(&sm.part[row]);
      for (uint32_t j = 0; j < C; ++j) {  // fixed order: deterministic and identical in all CTAs
        const float2 v = ld_cluster_f32x2(mapa_shared(my, j));
        la = __fadd_rn(la, v.x);
        lk = __fadd_rn(lk, v.y);
      }
      const float s = (lk == 0.f) ? 1.f : __fdiv_rn(la, lk);
      sm.srow[row] = s;
      if (p.row_scale != nullptr && rank == 0 && grow < p.M) p.row_scale[grow] = s;
    }
    if (do_lora && grow < p.M) {
      const uint32_t w = kLoraRank / C;
      __nv_bfloat16* trow = static_cast<__nv_bfloat16*>(p.t_out) + grow * kLoraRank + rank * w;
      for (uint32_t c = 0; c < w; c += 2) {
        float a0 = 0.f, a1 = 0.f;
        for (uint32_t j = 0; j < C; ++j) {
          a0 = __fadd_rn(a0, sm.recv[(j * 128 + row) * w + c]);
          a1 = __fadd_rn(a1, sm.recv[(j * 128 + row) * w + c + 1]);
        }
        *reinterpret_cast<__nv_bfloat162*>(trow + c) = __floats2bfloat162_rn(a0, a1);
      }
    }
  }

  __syncwarp();
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory

  if (warp == 1 && do_lora) tmem_dealloc(sm.tmem_base, kTmemCols);

  // ---- second sweep: compensated values (re-read what this thread wrote)
  if (do_sel && warp >= 2 && !sm.abort_flag) {
    const uint32_t half = (warp - 2) >> 2;
    const uint32_t row = 32 * (warp & 3) + lane;
    const int64_t grow = mb * 128 + row;
    if (grow < p.M) {
      const float s = sm.srow[row];
      uint4* vrow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.vals) + static_cast<size_t>(grow) * p.K);
      for (int b = 0; b < nboxes; ++b) {
        const int64_t kabs = kcol0 + 64 * b + 32 * half;
        uint4* d = vrow + (kabs >> 4);
        uint4 v0 = d[0], v1 = d[1];
        v0 = make_uint4(scale_pair(v0.x, s), scale_pair(v0.y, s), scale_pair(v0.z, s), scale_pair(v0.w, s));
        v1 = make_uint4(scale_pair(v1.x, s), scale_pair(v1.y, s), scale_pair(v1.z, s), scale_pair(v1.w, s));
        d[0] = v0;
        d[1] = v1;
      }
    }
  }
}

}  // namespace

int choose_sparsify_cluster(int64_t M, int64_t K, int num_sms) {
  const int64_t row_blocks = (M + 127) / 128;
  if (K % kMetaBlockK != 0) return 1;
  const int64_t kblocks = K / kMetaBlockK;
  int best = 1;
  for (int c = 2; c <= 8; c *= 2) {
    if (kblocks % c != 0) break;
    if (row_blocks * c > 2LL * num_sms) break;
    best = c;
  }
  return best;
}

cudaError_t launch_sparsify(const SparsifyLaunch& p, cudaStream_t stream) {
  const size_t smem = sizeof(SparsifySmem) + 1024;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(sparsify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.cluster), static_cast<unsigned>((p.M + 127) / 128), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sparsify_kernel, p);
}

}  // namespace lynx
