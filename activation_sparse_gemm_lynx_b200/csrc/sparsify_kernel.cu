// sparsify_kernel.cu -- online 2:4 activation sparsification with norm
// compensation, plus the LoRA down-projection T = X A^T from the same read of X.
//
// What it computes (RT-Lynx pages: qingkeai.online article sections 02-04;
// ai-feeds.com summary "core module 1"):
//   per token row m and group g of 4 consecutive K values: keep the 2 largest
//   magnitudes (ties to the lower index); L_all = sum|x|, L_kept = sum|kept|
//   (fp32); s = L_all / L_kept (1 if L_kept == 0); the kept values, 2 per
//   group in ascending position, and their 2-bit positions in the operand
//   layout of tcgen05.mma.sp; optionally T = X A^T (fp32 accumulate on tensor
//   cores).
//
// Three kernels:
//   sparsify_kernel  grid (C, ceil(M/128)): CTA (j, mb) covers rows
//                    [128 mb, 128 mb + 128) and dense columns [j K/C, (j+1) K/C).
//                    It writes the metadata and the kept values of its range
//                    (as they are, exact copies of X) and fp32 partials: the two
//                    row sums of its range and, with LoRA, T over its range.
//   finalize_kernel  per row: combines the C partials in a fixed order
//                    (deterministic) into s and T, written as bf16(T / s) when
//                    the GEMM applies s to its accumulator row (so that
//                    s * (S0 W^T + (T/s) B^T) = S(X) W^T + T B^T), else bf16(T).
//   rescale_kernel   standalone S(X): kept values v -> bf16(v * s).
//
// sparsify_kernel, per CTA (2 CTAs per SM):
//   warp 0      TMA producer: 128x64 tiles of X (and r x 64 tiles of A) into a
//               3-stage ring (128-byte swizzle, the UMMA K-major layout)
//   warp 1      owns TMEM (r columns, rounded up to a power of two), issues
//               tcgen05.mma M=128,N=r,K=16 on each X tile for the LoRA
//               down-projection
//   warps 2-9   256 row threads: thread = (row, half of each 64-wide tile,
//               i.e. 32 columns = 8 groups = two 16-bit metadata fields); the
//               kept values of a tile leave through one TMA store.  (Half rows
//               rather than quarter rows: half the synchronisation per element,
//               measured slightly faster than twice the threads.)
//
// Metadata layout (consumed by tcgen05.cp.128x128b + tcgen05.mma.sp kind::f16,
// M=128): one 2048-byte block per 128 rows x 128 dense K, 128 TMEM lanes x 16
// bytes.  Row m, dense column k (both within the block): lane = (m & 7) +
// 8*((k >> 4) & 1) + 16*(m >> 4), 32-bit word k >> 5, bit (k & 15) +
// 16*((m >> 3) & 1); 4 bits per group: lo | hi << 2.  Blocks are ordered row
// block major: block (mb, kb) starts at byte (mb * ceil(K/128) + kb) * 2048.
#include <cuda_bf16.h>

#include <algorithm>

#include "lynx_internal.h"
#include "lynx_ptx.cuh"
#include "lynx_select.cuh"

namespace lynx {

namespace {

constexpr int kStages = 3;
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = 32 * kComputeWarps;  // 256
constexpr int kThreads = 64 + kComputeThreads;        // 320
constexpr uint32_t kXTileBytes = 128 * 64 * 2;        // 16 KB
constexpr uint32_t kStoreTileBytes = 128 * 32 * 2;    // 8 KB: 128 rows x 32 kept values
constexpr uint32_t kBarCompute = 1;                   // named barrier of the row threads

// Shared memory, laid out at run time (the A ring depends on the LoRA rank r):
//   xring  kStages x 16 KB       X boxes, 128 rows x 64 columns (128-byte swizzle)
//   aring  kStages x r*128 B     A boxes, r rows x 64 columns (with LoRA only)
//   vstage 2 x 8 KB              kept values of one box (64-byte swizzle)
//   ctl    SparsifyCtl           barriers and per-row partials
// Every tile starts on a 1024-byte boundary (r % 16 == 0 makes r*128 a
// multiple of 2048).
struct SparsifyCtl {
  uint32_t sel_table[64];      // selection code -> kept-pair byte selector | nibble << 16
  float2 half1[128];           // partial sums of the second half of each row
  uint64_t full[kStages];
  uint64_t empty[kStages];     // row threads done with a stage (one arrival per warp)
  uint64_t mma_done[kStages];  // the LoRA MMAs done with a stage (tcgen05.commit)
  uint64_t vfree[2];           // a value staging buffer has been read by its TMA store
  uint64_t tdone;
  uint64_t drain;
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

struct SparsifyLayout {
  uint32_t a_tile;  // bytes of one A box (0 without LoRA)
  uint32_t aring, vstage, ctl, total;
};

__host__ __device__ inline SparsifyLayout sparsify_layout(bool lora, int r) {
  SparsifyLayout l;
  l.a_tile = lora ? static_cast<uint32_t>(r) * 128u : 0u;
  l.aring = kStages * kXTileBytes;
  l.vstage = l.aring + kStages * l.a_tile;
  l.ctl = l.vstage + 2 * kStoreTileBytes;
  l.total = l.ctl + static_cast<uint32_t>(sizeof(SparsifyCtl));
  return l;
}

// TMEM columns for the LoRA-down accumulator: a power of two >= 32 and >= r
__host__ __device__ inline uint32_t lora_tmem_cols(int r) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(r)) c <<= 1;
  return c;
}

// Top-2 of the 4 bf16 values in (w0 = x1:x0, w1 = x3:x2) by magnitude, ties to
// the lower index, together with the group's terms of the row's two L1 sums:
// |x0|, |x2| to la_even and |x1|, |x3| to la_odd, the kept magnitudes to lk_lo
// and lk_hi.  Returns the nibble lo | hi << 2 and the kept pair packed (x_lo in
// the low half).
__device__ __forceinline__ uint32_t select_group(uint32_t w0, uint32_t w1, const uint32_t* table,
                                                 uint32_t& kept, float& la_even, float& la_odd,
                                                 float& lk_lo, float& lk_hi) {
  const uint32_t a0 = w0 & 0x7FFF7FFFu;  // |x1| : |x0|
  const uint32_t a1 = w1 & 0x7FFF7FFFu;  // |x3| : |x2|
  add_bf16_pair(la_even, la_odd, a0);
  add_bf16_pair(la_even, la_odd, a1);
  const uint32_t ent = table[selection_code(a0, a1)];
  kept = __byte_perm(w0, w1, ent);
  add_bf16_pair(lk_lo, lk_hi, __byte_perm(a0, a1, ent));
  return ent >> 16;
}

__device__ __forceinline__ uint32_t scale_pair(uint32_t w, float s) {
  const float a = __fmul_rn(__uint_as_float(w << 16), s);
  const float b = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), s);
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void set_abort(SparsifyCtl& sm, uint32_t* status, uint32_t code) {
  record_error(status, code);
  sm.abort_flag = 1u;
}

__global__ void __launch_bounds__(kThreads, 2)
sparsify_kernel(const __grid_constant__ SparsifyLaunch p) {
  extern __shared__ uint8_t smem_raw[];
  const bool do_sel = (p.mode & kModeSelect) != 0;
  const bool do_lora = (p.mode & kModeLora) != 0;
  const bool write_out = do_sel && (p.mode & kModeNoOut) == 0;  // values and metadata leave
  const SparsifyLayout lay = sparsify_layout(do_lora, p.r);
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SparsifyCtl& sm = *reinterpret_cast<SparsifyCtl*>(base + lay.ctl);
  uint8_t* const xring = base;
  uint8_t* const aring = base + lay.aring;
  uint8_t* const vstage = base + lay.vstage;

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const uint32_t j = blockIdx.x;  // K range
  const int64_t mb = blockIdx.y;  // row block
  const int nboxes = p.boxes_per_cta;
  const int64_t kcol0 = static_cast<int64_t>(j) * nboxes * 64;
  const uint32_t tmem_cols = do_lora ? lora_tmem_cols(p.r) : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kComputeWarps);
      mbar_init(&sm.mma_done[s], 1);
    }
    for (int v = 0; v < 2; ++v) mbar_init(&sm.vfree[v], 1);
    mbar_init(&sm.tdone, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0u;
    fence_mbar_init();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 128) sm.sel_table[threadIdx.x - 64] = selection_table_entry(threadIdx.x - 64);
  // The first box's loads leave before the rest of the prologue (TMEM
  // allocation, the block barrier): its latency is the one nothing else hides.
  // The other stages' loads follow only once it has landed, so that the first
  // wave of requests from the whole grid is one box per CTA and each CTA can
  // start computing while the rest streams in.  The loads wait for the previous
  // kernel like every access to X below.
  const int preissued = (nboxes < 1) ? nboxes : 1;
  if (threadIdx.x == 0 && !p.stall_test) {
    tma_prefetch_desc(&p.tm_x);
    if (do_lora) tma_prefetch_desc(&p.tm_a);
    pdl_wait();
    const uint32_t tx = kXTileBytes + lay.a_tile;
    for (int b = 0; b < preissued; ++b) {
      mbar_arrive_expect_tx(&sm.full[b], tx);
      const int32_t kc = static_cast<int32_t>(kcol0 + 64 * b);
      tma_load_2d(xring + b * kXTileBytes, &p.tm_x, &sm.full[b], kc, static_cast<int32_t>(mb * 128));
      if (do_lora) tma_load_2d(aring + b * lay.a_tile, &p.tm_a, &sm.full[b], kc, 0);
    }
  }
  if (warp == 1 && do_lora) {
    tmem_alloc(&sm.tmem_base, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the prologue above may overlap the previous kernel on the stream; X (its
  // output, possibly) is read and this call's outputs (possibly still read by
  // it) are written only from here on
  pdl_wait();
  // the next kernel (finalize_kernel, or the GEMM that combines the partials
  // itself) may begin launching; it waits for this whole grid
  pdl_launch_dependents();
  // The GEMM of this call claims and publishes each row block through these
  // words; it reads them only after this grid has completed, and the previous
  // kernel on the stream (an earlier call's GEMM) has completed before here.
  if (p.fin_flags != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = static_cast<int>(threadIdx.x); i < p.fin_nflags; i += kThreads) p.fin_flags[i] = 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Loads box b into stage b % kStages once box b - kStages has left it.
    // The row threads' release of a stage also means that the kept values of
    // that box are staged, so the same thread then issues their TMA store and
    // hands back the buffer of the previous box's store, which has read it by
    // then (vfree).  The last box's buffer is not needed again.
    if (lane == 0) {
      if (write_out) tma_prefetch_desc(&p.tm_vals);
      const uint32_t tx = kXTileBytes + lay.a_tile;
      const bool store_rows = mb * 128 < p.M;  // a padding row block has metadata only
      bool ok = !p.stall_test;
      int issued = ok ? preissued : 0;
      for (int b = 0; ok && b < nboxes + kStages; ++b) {
        const int slot = b % kStages;
        if (sm.abort_flag) break;
        if (b >= kStages) {
          const int prev = b - kStages;  // the box that last used `slot`
          const uint32_t pph = static_cast<uint32_t>(prev / kStages) & 1u;
          if (do_sel) {
            if (!mbar_wait(&sm.empty[slot], pph)) {
              set_abort(sm, p.status, kDevTimeoutEmpty);
              break;
            }
            if (!write_out) {
              // nothing staged: the stage is free once the row threads are done
            } else if (store_rows) {
              tma_store_2d(&p.tm_vals, vstage + (prev & 1) * kStoreTileBytes,
                           static_cast<int32_t>((kcol0 + 64 * prev) / 2),
                           static_cast<int32_t>(mb * 128));
              bulk_commit();
              // the store of box prev - 1 has read its buffer (this one may still
              // be reading): hand that buffer back, without waiting on this store
              bulk_wait_read_le1();
              if (prev > 0) mbar_arrive(&sm.vfree[(prev - 1) & 1]);
            } else {
              mbar_arrive(&sm.vfree[prev & 1]);
            }
          }
          if (do_lora && !mbar_wait(&sm.mma_done[slot], pph)) {
            set_abort(sm, p.status, kDevTimeoutEmpty);
            break;
          }
        }
        if (b == preissued && b < kStages && preissued > 0 && !mbar_wait(&sm.full[0], 0)) {
          set_abort(sm, p.status, kDevTimeoutFull);
          break;
        }
        if (b >= preissued && b < nboxes) {
          mbar_arrive_expect_tx(&sm.full[slot], tx);
          const int32_t kc = static_cast<int32_t>(kcol0 + 64 * b);
          tma_load_2d(xring + slot * kXTileBytes, &p.tm_x, &sm.full[slot], kc,
                      static_cast<int32_t>(mb * 128));
          if (do_lora) tma_load_2d(aring + slot * lay.a_tile, &p.tm_a, &sm.full[slot], kc, 0);
          ++issued;
        }
      }
      bulk_wait_all();  // every value tile is in global memory
      // never leave with copies in flight: wait for the last fill of each slot
      for (int b = issued - 1; b >= 0 && b >= issued - kStages; --b) {
        if (!mbar_wait(&sm.full[b % kStages], static_cast<uint32_t>(b / kStages) & 1u,
                       kWaitLimitNs / 4))
          record_error(p.status, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ LoRA-down MMA
    if (do_lora && lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, static_cast<uint32_t>(p.r), false);
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
        const uint32_t xa = smem_u32(xring + slot * kXTileBytes);
        const uint32_t aa = smem_u32(aring + slot * lay.a_tile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = make_sdesc(xa + 32 * kk, 16, 1024, kSw128);
          const uint64_t db = make_sdesc(aa + 32 * kk, 16, 1024, kSw128);
          mma_bf16(t_tmem, da, db, idesc, (b | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&sm.mma_done[slot]);
      }
      tc_commit(&sm.tdone);
      // fires once every MMA issued above has completed (used on every path)
      tc_commit(&sm.drain);
      if (!mbar_wait(&sm.drain, 0)) record_error(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (do_sel) {
    // ------------------------------------------------------------ row threads
    const uint32_t hf = (warp - 2) >> 2;      // which 32 columns of each tile
    const uint32_t row = 32 * (warp & 3) + lane;
    const int64_t grow = mb * 128 + row;
    // metadata: this thread's 32 columns form two 16-bit fields, in lanes 8
    // apart (64 16-bit words) of the same block and word
    const uint32_t meta_lane = (row & 7) + 16 * (row >> 4);
    const uint32_t meta_hsel = (row >> 3) & 1;
    uint16_t* meta_row_blocks =
        reinterpret_cast<uint16_t*>(p.meta + static_cast<size_t>(mb) * p.kblocks * kMetaBlockBytes);
    // where this thread's four 16-byte chunks sit in the tile (128-byte
    // swizzle), and its 16 kept values in the 64-byte-swizzled store tile
    const uint32_t sw = row & 7;
    const uint32_t ld_off0 = row * 128 + (((4 * hf + 0) ^ sw) << 4);
    const uint32_t ld_off1 = row * 128 + (((4 * hf + 1) ^ sw) << 4);
    const uint32_t ld_off2 = row * 128 + (((4 * hf + 2) ^ sw) << 4);
    const uint32_t ld_off3 = row * 128 + (((4 * hf + 3) ^ sw) << 4);
    const uint32_t s64 = (row >> 1) & 3;
    const uint32_t vst_off0 = row * 64 + (((2 * hf) ^ s64) << 4);
    const uint32_t vst_off1 = row * 64 + (((2 * hf + 1) ^ s64) << 4);
    // fp32 partial sums of |x| and |kept|, even and odd positions apart
    float la0 = 0.f, la1 = 0.f, lk0 = 0.f, lk1 = 0.f;
    // this thread's first metadata field of a box: block (kabs >> 7) of the
    // row block, 16-bit word lane*8 + ((kabs >> 5) & 3)*2 + hsel, kabs = its
    // first dense column (32-bit: K < 2^30).  From one box to the next kabs
    // grows by 64: within a 128-column block (bit 6 of kabs clear) the word
    // index grows by 4; across a block boundary by 1024 - 4.
    const uint32_t kabs0 = static_cast<uint32_t>(kcol0) + 32 * hf;
    uint16_t* meta_ptr = meta_row_blocks + ((kabs0 >> 7) << 10) + meta_lane * 8 + meta_hsel +
                         (((kabs0 >> 5) & 3u) << 1);
    uint32_t meta_hi_half = (kabs0 >> 6) & 1u;
    uint32_t slot = 0, phase = 0;
    for (int b = 0; b < nboxes; ++b) {
      bool ok = !sm.abort_flag;
      if (ok && !mbar_wait(&sm.full[slot], phase)) {
        set_abort(sm, p.status, kDevTimeoutFull);
        ok = false;
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* tile = xring + slot * kXTileBytes;
      const uint4 v0 = *reinterpret_cast<const uint4*>(tile + ld_off0);
      const uint4 v1 = *reinterpret_cast<const uint4*>(tile + ld_off1);
      const uint4 v2 = *reinterpret_cast<const uint4*>(tile + ld_off2);
      const uint4 v3 = *reinterpret_cast<const uint4*>(tile + ld_off3);
      uint32_t kw[8];
      const uint32_t* tab = sm.sel_table;
      const uint32_t n0 = select_group(v0.x, v0.y, tab, kw[0], la0, la1, lk0, lk1);
      const uint32_t n1 = select_group(v0.z, v0.w, tab, kw[1], la0, la1, lk0, lk1);
      const uint32_t n2 = select_group(v1.x, v1.y, tab, kw[2], la0, la1, lk0, lk1);
      const uint32_t n3 = select_group(v1.z, v1.w, tab, kw[3], la0, la1, lk0, lk1);
      const uint32_t n4 = select_group(v2.x, v2.y, tab, kw[4], la0, la1, lk0, lk1);
      const uint32_t n5 = select_group(v2.z, v2.w, tab, kw[5], la0, la1, lk0, lk1);
      const uint32_t n6 = select_group(v3.x, v3.y, tab, kw[6], la0, la1, lk0, lk1);
      const uint32_t n7 = select_group(v3.z, v3.w, tab, kw[7], la0, la1, lk0, lk1);
      if (write_out) {
        meta_ptr[0] = static_cast<uint16_t>(n0 + n1 * 16u + n2 * 256u + n3 * 4096u);
        meta_ptr[64] = static_cast<uint16_t>(n4 + n5 * 16u + n6 * 256u + n7 * 4096u);
        meta_ptr += meta_hi_half ? 1020 : 4;
        meta_hi_half ^= 1u;
        // the store of box b - 2 has read this staging buffer
        if (!mbar_wait(&sm.vfree[b & 1], static_cast<uint32_t>((b >> 1) & 1) ^ 1u)) {
          set_abort(sm, p.status, kDevTimeoutEmpty);
          ok = false;
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        uint8_t* const vbuf = vstage + (b & 1) * kStoreTileBytes;
        *reinterpret_cast<uint4*>(vbuf + vst_off0) = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        *reinterpret_cast<uint4*>(vbuf + vst_off1) = make_uint4(kw[4], kw[5], kw[6], kw[7]);
        fence_proxy_async_smem();
      }
      // release the stage only after everything derived from it has been
      // produced: an arrive does not wait for this warp's loads in flight
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
    }
    const float my_la = __fadd_rn(la0, la1);
    const float my_lk = __fadd_rn(lk0, lk1);
    if (hf > 0) sm.half1[row] = make_float2(my_la, my_lk);
    named_bar_sync(kBarCompute, kComputeThreads);
    if (hf == 0 && grow < p.M) {
      const float2 o = sm.half1[row];
      p.lpart[static_cast<size_t>(j) * p.M + grow] = make_float2(__fadd_rn(my_la, o.x), __fadd_rn(my_lk, o.y));
    }
  }

  // ---- T partial of this K range: TMEM -> registers -> global (fp32).  The 8
  // row warps share it: warps w and w + 4 read the same 32 TMEM lanes (rows)
  // and take alternate 16-column chunks, two chunks per wait.
  if (do_lora && warp >= 2) {
    const uint32_t row = 32 * (warp & 3) + lane;
    const int64_t grow = mb * 128 + row;
    const int first = static_cast<int>((warp - 2) >> 2);  // 0 for warps 2-5, 1 for warps 6-9
    const int chunks = p.r / 16;
    if (!sm.abort_flag && mbar_wait(&sm.tdone, 0)) {
      tc_fence_after();
      float4* dst = reinterpret_cast<float4*>(p.tpart + (static_cast<size_t>(j) * p.M + grow) * p.r);
      const uint32_t lane_base = sm.tmem_base + ((32u * (warp & 3)) << 16);
      for (int c = first; c < chunks; c += 4) {
        const bool two = c + 2 < chunks;
        uint32_t r[2][16];
        tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(16 * c), r[0]);
        if (two) tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(16 * (c + 2)), r[1]);
        tmem_ld_wait();
        if (grow < p.M) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && !two) break;
            const int col = 16 * (c + 2 * h);
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              dst[(col + e) / 4] = make_float4(__uint_as_float(r[h][e]), __uint_as_float(r[h][e + 1]),
                                               __uint_as_float(r[h][e + 2]), __uint_as_float(r[h][e + 3]));
          }
        }
      }
      tc_fence_before();
    } else if (!sm.abort_flag) {
      set_abort(sm, p.status, kDevTimeoutAccum);
    }
  }

  __syncthreads();
  if (warp == 1 && do_lora) tmem_dealloc(sm.tmem_base, tmem_cols);
}

// One warp per row: s from the C partial sums, T from the C partial products
// (fixed order), T [M, r] written as bf16(T / s) when `divide`.
__global__ void __launch_bounds__(256)
finalize_kernel(const float2* __restrict__ lpart, const float* __restrict__ tpart, int64_t M,
                int C, int r, int do_scale, int do_lora, int divide, float* __restrict__ row_scale,
                __nv_bfloat16* __restrict__ t_out) {
  pdl_launch_dependents();
  pdl_wait();  // the partials of sparsify_kernel
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const uint32_t lane = threadIdx.x & 31u;
  if (row >= M) return;
  float s = 1.f;
  // all C partials are loaded before any is added (the loads overlap), then
  // summed in the fixed order j = 0, 1, ...
  if (do_scale) {
    float2 v[kMaxSplit];
#pragma unroll
    for (int j = 0; j < kMaxSplit; ++j)
      if (j < C) v[j] = __ldcg(lpart + static_cast<size_t>(j) * M + row);
    float la = 0.f, lk = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxSplit; ++j) {
      if (j < C) {
        la = __fadd_rn(la, v[j].x);
        lk = __fadd_rn(lk, v[j].y);
      }
    }
    s = (lk == 0.f) ? 1.f : __fdiv_rn(la, lk);
    if (lane == 0) row_scale[row] = s;
  }
  if (do_lora) {
    // columns 2c, 2c + 1 of each partial, c = lane, lane + 32, ...
    for (int c = static_cast<int>(lane); 2 * c < r; c += 32) {
      float2 v[kMaxSplit];
#pragma unroll
      for (int j = 0; j < kMaxSplit; ++j)
        if (j < C)
          v[j] = __ldcg(reinterpret_cast<const float2*>(tpart + (static_cast<size_t>(j) * M + row) * r) + c);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxSplit; ++j) {
        if (j < C) {
          a0 = __fadd_rn(a0, v[j].x);
          a1 = __fadd_rn(a1, v[j].y);
        }
      }
      if (divide) {
        a0 = __fdiv_rn(a0, s);
        a1 = __fdiv_rn(a1, s);
      }
      reinterpret_cast<__nv_bfloat162*>(t_out + row * r)[c] = __floats2bfloat162_rn(a0, a1);
    }
  }
}

// Standalone S(X): the kept values become bf16(v * s) in place.  One thread per
// 8 values (16 bytes); rows of K/2 values.
__global__ void __launch_bounds__(256)
rescale_kernel(uint4* __restrict__ vals, const float* __restrict__ row_scale, int64_t M,
               int64_t K) {
  pdl_wait();  // s from finalize_kernel, values from sparsify_kernel
  const int64_t per_row = K / 16;  // uint4 per row (K/2 bf16 = K bytes)
  const int64_t total = M * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float s = __ldg(row_scale + i / per_row);
    const uint4 v = vals[i];
    vals[i] = make_uint4(scale_pair(v.x, s), scale_pair(v.y, s), scale_pair(v.z, s), scale_pair(v.w, s));
  }
}

}  // namespace

size_t sparsify_smem_bytes(int mode, int r) {
  return sparsify_layout((mode & kModeLora) != 0, r).total + 1024;  // + alignment slack
}

// K ranges per row block: the largest C <= kMaxSplit dividing the 64-column
// boxes of a row such that C * ceil(M/128) CTAs fit in one wave (2 per SM).
int choose_sparsify_split(int64_t M, int64_t K, int num_sms) {
  const int64_t row_blocks = meta_row_blocks(M);
  const int64_t boxes = K / 64;
  int best = 1;
  for (int c = 2; c <= kMaxSplit; ++c) {
    if (boxes % c != 0) continue;
    if (row_blocks * c > 2LL * num_sms) break;
    best = c;
  }
  return best;
}

cudaError_t launch_sparsify(const SparsifyLaunch& p, cudaStream_t stream) {
  const size_t smem = sparsify_smem_bytes(p.mode, p.r);
  // the largest layout (r = kLoraRankMax) is allowed once per device
  static std::once_flag once[64];
  static cudaError_t configured[64];
  cudaError_t e = once_per_device(once, configured, []() {
    return cudaFuncSetAttribute(sparsify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sparsify_smem_bytes(kModeSelect | kModeLora, kLoraRankMax)));
  });
  if (e != cudaSuccess) return e;
  // metadata row blocks come in pairs: the block past M (if any) gets the
  // pattern of all-zero rows, so a CTA pair of the GEMM never reads garbage
  const dim3 grid(static_cast<unsigned>(p.split), static_cast<unsigned>(meta_row_blocks(p.M)), 1);
  e = launch_after_previous(sparsify_kernel, grid, dim3(kThreads), smem, stream, p);
  if (e != cudaSuccess || p.skip_finalize) return e;
  const bool do_sel = (p.mode & kModeSelect) != 0;
  const bool do_lora = (p.mode & kModeLora) != 0;
  const bool scaled = (p.mode & kModeScaled) != 0;
  const unsigned fin_blocks = static_cast<unsigned>((p.M + 7) / 8);
  e = launch_after_previous(finalize_kernel, dim3(fin_blocks), dim3(256), 0, stream,
                            static_cast<const float2*>(p.lpart), static_cast<const float*>(p.tpart),
                            p.M, p.split, p.r, do_sel ? 1 : 0, do_lora ? 1 : 0,
                            (do_sel && !scaled) ? 1 : 0, p.row_scale,
                            static_cast<__nv_bfloat16*>(p.t_out));
  if (e != cudaSuccess || !(do_sel && scaled)) return e;
  const int64_t n16 = p.M * (p.K / 16);
  const unsigned rb = static_cast<unsigned>(std::min<int64_t>((n16 + 255) / 256, 4096));
  return launch_after_previous(rescale_kernel, dim3(rb), dim3(256), 0, stream,
                               static_cast<uint4*>(p.vals), static_cast<const float*>(p.row_scale),
                               p.M, p.K);
}

}  // namespace lynx
