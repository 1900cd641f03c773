// gemm_pair_kernel.cu -- the Lynx GEMM on CTA pairs (tcgen05 cta_group::2):
//   Y[M,N] = bf16( act( s_row * (S(X) W^T + T' B^T) + bias ) )   (act: none or GELU)
// Same arithmetic as gemm_kernel.cu (see there and the RT-Lynx references),
// computed on 256 x 256 output tiles by a pair of CTAs on the two SMs of a
// TPC: each CTA holds 128 rows of A (compressed activations, or X on the dense
// path) and 128 of the 256 rows of the W tile in its own shared memory; one
// tcgen05.mma(.sp).cta_group::2 with M = 256, N = 256 issued by the leader CTA
// reads both halves, and each CTA's TMEM receives its 128 rows of the
// accumulator.  Splitting B across the pair halves the operand bytes each SM
// must stage per MMA, which is what the 2:4 sparse rate (twice the dense rate
// per byte of B) needs.
//
// Per CTA (both CTAs run the same roles):
//   warp 0      TMA producer: own 128 rows of A (and of the LoRA T), own 128
//               rows of W (and of the LoRA B); on the sparse path one 2 KB
//               metadata block (own 128 rows) per stage.  All loads
//               complete on the leader's "full" barrier (cta_group::2 form, no
//               multicast); the leader arms it with both CTAs' bytes.
//   warp 1      TMEM (pair allocation, 512 columns); in the leader CTA the
//               single MMA issuer: tcgen05.cp of both CTAs' metadata, the MMAs,
//               and commits multicast to both CTAs' "empty" / "acc_full"
//               barriers.
//   warps 2-9   epilogue on the CTA's own 128 accumulator rows: act(s * acc + bias)
//               -> bf16 -> global; releases the accumulator by arriving on the
//               leader's "acc_empty" barrier.
//   warp 10     in the leader CTA: waits for each filled stage ("full") and
//               hands it to the MMA issuer through a named barrier.  A
//               shared-memory barrier poll in the issuing warp itself costs the
//               tensor pipe about a fifth of its rate when the operands change
//               from stage to stage; a hardware barrier between two warps does
//               not.
#include <cuda_bf16.h>

#include "lynx_act.cuh"
#include "lynx_internal.h"
#include "lynx_ptx.cuh"
#include "lynx_select.cuh"

namespace lynx {

namespace {

constexpr int kThreads = 352;
constexpr uint32_t kHelperWarp = 10;
constexpr uint32_t kBarStage0 = 3;  // named barriers 3 .. 3 + stages - 1: stage hand-off
constexpr uint32_t kHandoffThreads = 64;  // the MMA warp and the helper warp
constexpr uint32_t kTmemCols = 512;
constexpr int kEslots = 4;
constexpr uint32_t kBarEpilogue = 2;
constexpr uint32_t kEpiThreads = 256;
constexpr uint16_t kPairMask = 0x3;

// One pipeline stage covers 128 dense K: on the sparse path A is 128 rows x 64
// kept values (one 128-byte-row tile), W two 128 x 64 tiles, plus one 2 KB
// metadata block (4 stages fit); on the dense path A and W are two 128 x 64
// tiles each (3 stages fit).  Fewer, larger stages measured faster on the dense
// path (8 MMAs per hand-off instead of 4); on the sparse path 4 stages of 4 MMAs
// beat 2 stages of 8.  LoRA stages (K = 32 each) reuse the A / B slots with
// 64-byte-row tiles.
// FUSED (sparse): the stage holds the dense X tile (two 128 x 64 tiles); the
// epilogue warps compress it in place into the first one, which is then the
// MMA's A operand, and write the metadata block.
template <bool SPARSE, bool FUSED = false>
struct PairCfg {
  static constexpr int kBK = 128;
  static constexpr uint32_t kABytes = SPARSE ? 128u * 128u : 2u * 128u * 128u;  // own 128 rows
  static constexpr uint32_t kXBytes = FUSED ? 2u * 128u * 128u : 0u;  // dense X tile (fused)
  static constexpr uint32_t kBOff = FUSED ? kXBytes : kABytes;        // W tile
  static constexpr uint32_t kBBytes = 128u * static_cast<uint32_t>(kBK) * 2u;  // own 128 W rows
  static constexpr uint32_t kEOff = kBOff + kBBytes;                   // metadata block
  static constexpr uint32_t kEBytes = SPARSE ? 2048u : 0u;
  static constexpr uint32_t kStageBytes = ((kEOff + kEBytes + 1023u) / 1024u) * 1024u;
  // of the 227 KB: 16 KB epilogue store staging, ~3 KB barriers / bias / alignment
  static constexpr int kStagesFit = static_cast<int>((208u * 1024u) / kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr uint32_t kEcol0 = 256;
  static constexpr uint32_t kLoraABytes = 128u * 64u;  // T: own 128 rows x 32
  static constexpr uint32_t kLoraBBytes = 128u * 64u;  // B: own 128 rows x 32
  static_assert(kStages >= 3, "pipeline too shallow");
  static_assert(kBarStage0 + kStages <= 16, "named barriers");
  static_assert(!FUSED || SPARSE, "the fused variant is sparse");
};

template <bool SPARSE, bool FUSED = false>
struct __align__(1024) PairSmem {
  using C = PairCfg<SPARSE, FUSED>;
  uint8_t stage[C::kStages][C::kStageBytes];
  uint8_t ystage[8][2][1024];  // per epilogue warp: two 32 rows x 16 columns bf16 tiles (32B swizzle)
  uint64_t full[C::kStages];   // used in the leader CTA
  uint64_t empty[C::kStages];  // each CTA's producer waits on its own
  uint64_t acc_full;           // each CTA's epilogue waits on its own
  uint64_t acc_empty;          // used in the leader CTA (both CTAs' epilogues arrive)
  uint64_t drain;
  uint64_t rows_ready;         // the rows of T of all this CTA's tiles are combined (fused, LoRA)
  uint64_t xfull[C::kStages];  // FUSED: this CTA's X tile of the stage has landed
  uint64_t afull[C::kStages];  // FUSED (leader): both CTAs' compressed A and metadata are written
  uint32_t sel_table[64];      // FUSED: selection code -> kept-pair byte selector | nibble << 16
  float bias_s[256];
  uint32_t tmem_base;
  uint32_t own_claimed[32];    // fused combining: which of the CTA's own slices it claimed
  int open_slice;              // fused combining: an open slice found in the round of checks
  volatile uint32_t abort_flag;
};

// s of row `row` from the sparsify pass's K-range partials, summed in the fixed
// order j = 0, 1, ...: the same arithmetic as finalize_kernel.
__device__ __forceinline__ float row_scale_from_partials(const float2* lpart, int64_t M, int split,
                                                         int64_t row) {
  float2 v[kMaxSplit];
#pragma unroll
  for (int j = 0; j < kMaxSplit; ++j)
    if (j < split) v[j] = __ldcg(lpart + static_cast<size_t>(j) * M + row);
  float la = 0.f, lk = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxSplit; ++j) {
    if (j < split) {
      la = __fadd_rn(la, v[j].x);
      lk = __fadd_rn(lk, v[j].y);
    }
  }
  return (lk == 0.f) ? 1.f : __fdiv_rn(la, lk);
}

// tiles walk M first inside a group of `group_m` pair-rows (sized on the host so
// that the group's A rows stay resident in L2 while W streams once per group)
__device__ __forceinline__ void pair_tile_coords(int tile, int ntm2, int ntn, int group_m, int& pm,
                                                 int& nb) {
  const int per_group = group_m * ntn;
  const int group = tile / per_group;
  const int first = group * group_m;
  const int gm = min(group_m, ntm2 - first);
  const int in_group = tile - group * per_group;
  pm = first + in_group % gm;
  nb = in_group / gm;
}

// Rows of the sparsify pass's partials are combined in slices of 32 rows: s
// (fin_mode 1) and, with LoRA, T summed over the K ranges in the fixed order
// j = 0, 1, ... and written as bf16(T / s) (fin_mode 1) or bf16(T) (fin_mode
// 2).  256 threads, 8 per row; each takes the row's 8-column chunks sub, sub +
// 8, ... of r / 8.
constexpr int kSliceRows = 32;
constexpr int kMaxOwnSlices = 32;

__device__ __forceinline__ void combine_slice(const GemmLaunch& p, int sl, uint32_t et) {
  const int64_t row = static_cast<int64_t>(sl) * kSliceRows + (et >> 3);
  if (row >= p.M) return;
  const uint32_t sub = et & 7u;
  const int chunks = p.lora ? p.r / 8 : 0;
  float s = 1.f;
  if (p.fin_mode == 1) {
    s = row_scale_from_partials(p.fin_lpart, p.M, p.fin_split, row);
    if (sub == 0) p.fin_scale[row] = s;
  }
  for (int q = static_cast<int>(sub); q < chunks; q += 8) {
    float4 v[kMaxSplit][2];
#pragma unroll
    for (int j = 0; j < kMaxSplit; ++j) {
      if (j < p.fin_split) {
        const float4* src = reinterpret_cast<const float4*>(
            p.fin_tpart + (static_cast<size_t>(j) * p.M + row) * p.r + 8 * q);
        v[j][0] = __ldcg(src);
        v[j][1] = __ldcg(src + 1);
      }
    }
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxSplit; ++j) {
      if (j < p.fin_split) {
        a[0] = __fadd_rn(a[0], v[j][0].x);
        a[1] = __fadd_rn(a[1], v[j][0].y);
        a[2] = __fadd_rn(a[2], v[j][0].z);
        a[3] = __fadd_rn(a[3], v[j][0].w);
        a[4] = __fadd_rn(a[4], v[j][1].x);
        a[5] = __fadd_rn(a[5], v[j][1].y);
        a[6] = __fadd_rn(a[6], v[j][1].z);
        a[7] = __fadd_rn(a[7], v[j][1].w);
      }
    }
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0 = a[2 * e], x1 = a[2 * e + 1];
      if (p.fin_mode == 1) {
        x0 = __fdiv_rn(x0, s);
        x1 = __fdiv_rn(x1, s);
      }
      __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
      pk[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.fin_t) + row * p.r + 8 * q) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// After combining a slice: its s and T are read by other CTAs (generic loads)
// and by TMA (async proxy); thread 0 then publishes the slice as done.
__device__ __forceinline__ void publish_slices_fence() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
}

__device__ __forceinline__ void store_release(uint32_t* flag, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t load_acquire(const uint32_t* flag) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  return v;
}

// Before its first tile, the epilogue warps of a CTA make sure that every row
// of its tiles is combined.  Each 32-row slice has a state word: 0 open, 1
// claimed by a CTA that is combining it, 2 done.  First every CTA claims and
// combines the slices it owns (slice i belongs to CTA i mod grid, so the work
// is spread evenly); then it checks the slices of its own tiles in one round of
// acquiring loads, claims and combines any that is still open (its owner has
// not started), and waits (bounded) only for slices that a running CTA has
// claimed.  So no CTA waits for one that has not started (the grid needs no
// co-residency), and the words start at 0 in every call (the sparsify pass of
// the same call clears them), so neither an earlier call nor a replayed graph
// can leave a stale "done".  Returns false (in every thread) if a wait ran out.
template <typename Smem>
__device__ __noinline__ bool ensure_rows_of_tiles(const GemmLaunch& p, Smem& sm, uint32_t et, int ntm2,
                                                  int ntn, int first_tile, int tile_step, int ntiles,
                                                  uint32_t rank) {
  const int nsl = static_cast<int>((p.M + kSliceRows - 1) / kSliceRows);
  const int cta = static_cast<int>(blockIdx.x);
  const int grid = static_cast<int>(gridDim.x);
  // 1. the slices this CTA owns
  const int nown = cta < nsl ? min(kMaxOwnSlices, (nsl - cta + grid - 1) / grid) : 0;
  if (et < static_cast<uint32_t>(nown))
    sm.own_claimed[et] = atomicCAS(p.fin_flags + cta + static_cast<int>(et) * grid, 0u, 1u) == 0u ? 1u : 0u;
  named_bar_sync(kBarEpilogue, kEpiThreads);
  bool any_own = false;
  for (int k = 0; k < nown; ++k) {
    if (sm.own_claimed[k]) {
      combine_slice(p, cta + k * grid, et);
      any_own = true;
    }
  }
  if (any_own) {
    publish_slices_fence();
    named_bar_sync(kBarEpilogue, kEpiThreads);
    if (et < static_cast<uint32_t>(nown) && sm.own_claimed[et])
      store_release(p.fin_flags + cta + static_cast<int>(et) * grid, 2u);
  }
  // 2. the slices of this CTA's tiles: entry e = (tile index e / 4, slice e % 4
  // of the tile's 128-row block of this CTA)
  const int mine = first_tile < ntiles ? (ntiles - first_tile + tile_step - 1) / tile_step : 0;
  const int entries = 4 * mine;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    bool pending = false;
    int open = -1;
    for (int e = static_cast<int>(et); e < entries; e += kEpiThreads) {
      int pm, nb;
      pair_tile_coords(first_tile + (e >> 2) * tile_step, ntm2, ntn, p.group_m, pm, nb);
      const int sl = (pm * 2 + static_cast<int>(rank)) * 4 + (e & 3);
      if (sl >= nsl) continue;
      const uint32_t v = load_acquire(p.fin_flags + sl);
      if (v != 2u) pending = true;
      if (v == 0u) open = sl;
    }
    if (et == 0) sm.open_slice = -1;
    named_bar_sync(kBarEpilogue, kEpiThreads);
    if (open >= 0) atomicMax(&sm.open_slice, open);
    if (!named_bar_red_or(kBarEpilogue, kEpiThreads, pending)) return true;
    const int sl = sm.open_slice;
    if (sl >= 0) {
      // an open slice: its owner has not got this far; combine it here
      if (et == 0) sm.own_claimed[0] = atomicCAS(p.fin_flags + sl, 0u, 1u) == 0u ? 1u : 0u;
      named_bar_sync(kBarEpilogue, kEpiThreads);
      if (sm.own_claimed[0]) {
        combine_slice(p, sl, et);
        publish_slices_fence();
        named_bar_sync(kBarEpilogue, kEpiThreads);
        if (et == 0) store_release(p.fin_flags + sl, 2u);
      }
    } else {
      __nanosleep(256);
    }
    const bool late = globaltimer_ns() - t0 > kWaitLimitNs;
    if (named_bar_red_or(kBarEpilogue, kEpiThreads, late)) return false;
  }
}

// FUSED: the epilogue warps turn the dense X tile of each main stage of one
// tile into the MMA's sparse operand, in place, and tell the leader (afull):
// thread et takes row et / 2 and half et % 2 of the stage's 128 K (16 groups of
// 4).  The compressed row (64 kept values) goes to the row's 128 bytes of the
// first X tile, in its 128-byte swizzle, which is the A layout of the sparse
// path; the nibbles go to the stage's metadata block in the operand layout of
// tcgen05.mma.sp (the same as the sparsify pass writes).  The two threads of a
// row are neighbouring lanes, and a warp reads all its X before it writes.
// LoRA stages only pass the barrier on.  `g` is the stage counter shared with
// the producer and the MMA issuer.  Returns false if a wait ran out (this
// warp's answer; the caller makes it common).
template <typename C, typename Smem>
__device__ __forceinline__ bool compress_tile_stages(Smem& sm, uint32_t& g, int nk, int steps, uint32_t et,
                                                     uint32_t lane) {
  const uint32_t r = et >> 1, h = et & 1u, sw = r & 7u;
  for (int kit = 0; kit < steps; ++kit, ++g) {
    const uint32_t slot = g % C::kStages;
    const uint32_t ph = (g / C::kStages) & 1u;
    bool ok = !sm.abort_flag && mbar_wait(&sm.xfull[slot], ph);
    if (!__all_sync(0xffffffffu, ok)) return false;
    if (kit < nk) {
      uint8_t* st = sm.stage[slot];
      const uint8_t* xrow = st + h * 16384u + r * 128u;
      uint4 v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = *reinterpret_cast<const uint4*>(xrow + ((c ^ sw) << 4));
      uint32_t kept[16], nib[16];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        nib[2 * c] = select_group_kept(v[c].x, v[c].y, sm.sel_table, kept[2 * c]);
        nib[2 * c + 1] = select_group_kept(v[c].z, v[c].w, sm.sel_table, kept[2 * c + 1]);
      }
      __syncwarp();  // the whole warp has read its X rows before any is overwritten
      uint8_t* arow = st + r * 128u;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(arow + (((4u * h + i) ^ sw) << 4)) =
            make_uint4(kept[4 * i], kept[4 * i + 1], kept[4 * i + 2], kept[4 * i + 3]);
      // 16-bit field of (row r, 16-K chunk c16): lane (r%8) + 8(c16%2) + 16(r/16),
      // 32-bit word c16/2, upper half for rows with (r/8) odd
      uint16_t* e = reinterpret_cast<uint16_t*>(st + C::kEOff);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t c16 = 4u * h + i;
        const uint32_t tl = (r & 7u) + 8u * (c16 & 1u) + 16u * (r >> 4);
        e[tl * 8u + (c16 >> 1) * 2u + ((r >> 3) & 1u)] =
            static_cast<uint16_t>(nib[4 * i] + nib[4 * i + 1] * 16u + nib[4 * i + 2] * 256u + nib[4 * i + 3] * 4096u);
      }
      fence_proxy_async_smem();  // the MMA reads them through the async proxy
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster_release(mapa_shared(smem_u32(&sm.afull[slot]), 0));
  }
  return true;
}

template <bool SPARSE, int ACT, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
lynx_gemm_pair_kernel(const __grid_constant__ GemmLaunch p) {
  using C = PairCfg<SPARSE, FUSED>;
  extern __shared__ uint8_t smem_raw[];
  PairSmem<SPARSE, FUSED>& sm = *reinterpret_cast<PairSmem<SPARSE, FUSED>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int ntm2 = static_cast<int>((p.M + 255) / 256);
  const int ntn = static_cast<int>((p.N + 255) / 256);
  const int ntiles = ntm2 * ntn;
  const int cluster_id = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);
  const int nk = static_cast<int>(p.K / C::kBK);
  const int kblocks = static_cast<int>((p.K + 127) / 128);
  const bool lora = p.lora != 0;
  const int lsteps = lora ? (p.r + 31) / 32 : 0;  // LoRA-up stages of K = 32 (zero-filled past r)
  const int steps = nk + lsteps;
  const bool fused = p.fin_mode != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 2 * 8);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.rows_ready, 1);
    if (FUSED) {
      for (int s = 0; s < C::kStages; ++s) {
        mbar_init(&sm.xfull[s], 1);
        mbar_init(&sm.afull[s], 2 * 8);  // the 8 epilogue warps of both CTAs
      }
    }
    sm.abort_flag = 0u;
    fence_mbar_init();
  }
  if (FUSED && threadIdx.x >= 64 && threadIdx.x < 128)
    sm.sel_table[threadIdx.x - 64] = selection_table_entry(threadIdx.x - 64);
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before any cross-CTA signal
  tc_fence_after();
  // the prologue above may overlap the previous kernel (programmatic launch);
  // its outputs (compressed values, metadata, s, T) are read only from here on
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_b);
      if (SPARSE) tma_prefetch_desc(&p.tm_e);
      if (lora) {
        tma_prefetch_desc(&p.tm_t);
        tma_prefetch_desc(&p.tm_lb);
      }
      uint32_t g = 0;
      bool ok = !p.stall_test;
      bool rows_ready = !fused;
      for (int tile = cluster_id; ok && tile < ntiles; tile += nclusters) {
        int pm, nb;
        pair_tile_coords(tile, ntm2, ntn, p.group_m, pm, nb);
        const int32_t row0 = pm * 256 + static_cast<int32_t>(rank) * 128;
        const int32_t col0 = nb * 256 + static_cast<int32_t>(rank) * 128;
        const int mb = pm * 2 + static_cast<int>(rank);  // this CTA's 128-row block
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
          const uint32_t lead_full = mapa_shared(smem_u32(&sm.full[slot]), 0);
          if (FUSED && kit < nk) {
            // this CTA's dense X tile into its own shared memory (own barrier);
            // the W tile as on the sparse path
            mbar_arrive_expect_tx(&sm.xfull[slot], C::kXBytes);
            tma_load_2d(st, &p.tm_a, &sm.xfull[slot], kit * C::kBK, row0);
            tma_load_2d(st + 16384, &p.tm_a, &sm.xfull[slot], kit * C::kBK + 64, row0);
            if (leader) mbar_arrive_expect_tx(&sm.full[slot], 2u * C::kBBytes);
            tma_load_2d_pair(st + C::kBOff, &p.tm_b, lead_full, kit * C::kBK, col0);
            tma_load_2d_pair(st + C::kBOff + 16384, &p.tm_b, lead_full, kit * C::kBK + 64, col0);
          } else if (kit < nk) {
            if (leader) mbar_arrive_expect_tx(&sm.full[slot], 2u * (C::kABytes + C::kBBytes + C::kEBytes));
            // A: 64 kept values (sparse) or 64 dense values (dense) per row
            if (SPARSE) {
              tma_load_2d_pair(st, &p.tm_a, lead_full, kit * 64, row0);
            } else {
              tma_load_2d_pair(st, &p.tm_a, lead_full, kit * C::kBK, row0);
              tma_load_2d_pair(st + 16384, &p.tm_a, lead_full, kit * C::kBK + 64, row0);
            }
            tma_load_2d_pair(st + C::kBOff, &p.tm_b, lead_full, kit * C::kBK, col0);
            tma_load_2d_pair(st + C::kBOff + 16384, &p.tm_b, lead_full, kit * C::kBK + 64, col0);
            if (SPARSE) {
              // metadata block (mb, kit): 2 KB seen as 8 rows of 256 bytes
              tma_load_2d_pair(st + C::kEOff, &p.tm_e, lead_full, 0, (mb * kblocks + kit) * 8);
            }
          } else {
            const int l = kit - nk;
            if (!rows_ready) {
              // the rows of T of every tile of this CTA are combined (the
              // epilogue warps saw it)
              if (sm.abort_flag || !mbar_wait(&sm.rows_ready, 0)) {
                if (!sm.abort_flag) {
                  record_error(p.status, kDevTimeoutFinalize);
                  sm.abort_flag = 1u;
                }
                ok = false;
                break;
              }
              if (sm.abort_flag) {
                ok = false;
                break;
              }
              asm volatile("fence.proxy.async.global;" ::: "memory");  // T is then read by TMA
              rows_ready = true;
            }
            if (FUSED) mbar_arrive(&sm.xfull[slot]);  // no X in a LoRA stage: the phase just passes
            if (leader) mbar_arrive_expect_tx(&sm.full[slot], 2u * (C::kLoraABytes + C::kLoraBBytes));
            tma_load_2d_pair(st, &p.tm_t, lead_full, l * 32, row0);
            tma_load_2d_pair(st + C::kBOff, &p.tm_lb, lead_full, l * 32, col0);
          }
        }
      }
      // fused: this CTA's last X loads have landed (normally already consumed)
      if (FUSED) {
        for (uint32_t b = g; b > 0 && b + C::kStages > g; --b) {
          const uint32_t x = b - 1;
          if (!mbar_wait(&sm.xfull[x % C::kStages], (x / C::kStages) & 1u, kWaitLimitNs / 4))
            record_error(p.status, kDevTimeoutDrain);
        }
      }
      // drain (leader): the last fill of every stage, both CTAs' bytes, has landed
      if (leader) {
        const uint32_t issued = g;
        for (uint32_t b = issued; b > 0 && b + C::kStages > issued; --b) {
          const uint32_t x = b - 1;
          if (!mbar_wait(&sm.full[x % C::kStages], (x / C::kStages) & 1u, kWaitLimitNs / 4))
            record_error(p.status, kDevTimeoutDrain);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    // The whole warp runs the loop (operands stay warp-uniform); one elected
    // lane issues each tcgen05 instruction.
    if (leader) {
      const uint32_t idesc_main = make_idesc_bf16(256, 256, SPARSE);
      const uint32_t idesc_dense = make_idesc_bf16(256, 256, false);
      uint32_t g = 0, eslot = 0;
      int acc_count = 0;
      bool stop = false;
      for (int tile = cluster_id; !stop && tile < ntiles; tile += nclusters, ++acc_count) {
        bool err = sm.abort_flag || !mbar_wait(&sm.acc_empty, (static_cast<uint32_t>(acc_count) & 1u) ^ 1u);
        err = __any_sync(0xffffffffu, err);
        if (err && lane == 0 && !sm.abort_flag) {
          record_error(p.status, kDevTimeoutAccum);
          sm.abort_flag = 1u;
        }
        tc_fence_after();
        const uint32_t d_tmem = sm.tmem_base;
        uint32_t accumulate = 0;
        for (int kit = 0; kit < steps; ++kit, ++g) {
          const uint32_t slot = g % C::kStages;
          // the helper warp says when stage g has landed; both warps leave
          // together (same barrier, same reduced flag) once either saw an error
          if (named_bar_red_or(kBarStage0 + slot, kHandoffThreads, err || sm.abort_flag)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm.stage[slot]);
          const uint32_t sb = sa + C::kBOff;
          if (kit < nk) {
            if (SPARSE) {
              eslot = (eslot + 1) % kEslots;
              const uint64_t edesc = make_sdesc(sa + C::kEOff, 2048, 128, kSwNone);
              if (elect_one()) tc_cp_128x128b_pair(sm.tmem_base + C::kEcol0 + 4 * eslot, edesc);
              __syncwarp();
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t ecol = C::kEcol0 + 4 * eslot + j;
                const uint64_t da = make_sdesc(sa + 32 * j, 16, 1024, kSw128);
                const uint64_t db = make_sdesc(sb + (j >> 1) * 16384 + 64 * (j & 1), 16, 1024, kSw128);
                if (elect_one())
                  mma_sp_bf16_pair(d_tmem, da, db, sm.tmem_base + (ecol & ~1u), idesc_main | (ecol & 1u),
                                   accumulate);
                __syncwarp();
                accumulate = 1;
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + 32 * (kk & 3);
                const uint64_t da = make_sdesc(sa + off, 16, 1024, kSw128);
                const uint64_t db = make_sdesc(sb + off, 16, 1024, kSw128);
                if (elect_one()) mma_bf16_pair(d_tmem, da, db, idesc_main, accumulate);
                __syncwarp();
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
              if (elect_one()) mma_bf16_pair(d_tmem, da, db, idesc_dense, accumulate);
              __syncwarp();
              accumulate = 1;
            }
          }
          if (elect_one()) tc_commit_pair_mc(&sm.empty[slot], kPairMask);
          __syncwarp();
        }
        if (stop) break;
        if (elect_one()) tc_commit_pair_mc(&sm.acc_full, kPairMask);
        __syncwarp();
      }
      if (elect_one()) tc_commit_pair_mc(&sm.drain, 0x1);
      __syncwarp();
      if (!mbar_wait(&sm.drain, 0) && lane == 0) record_error(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == kHelperWarp) {
    // ------------------------------------------------------------ stage hand-off (leader)
    // Walks the same (tile, stage) sequence as the MMA issuer: one barrier
    // round per stage, in the same order, so every round has both warps.
    if (leader) {
      uint32_t g = 0;
      bool stop = false;
      for (int tile = cluster_id; !stop && tile < ntiles; tile += nclusters) {
        for (int kit = 0; kit < steps; ++kit, ++g) {
          const uint32_t slot = g % C::kStages;
          const uint32_t ph = (g / C::kStages) & 1u;
          bool ok = !sm.abort_flag && mbar_wait(&sm.full[slot], ph);
          // fused: both CTAs' epilogue warps have compressed this stage's X
          if (FUSED) ok = ok && !sm.abort_flag && mbar_wait_cluster(&sm.afull[slot], ph);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok && lane == 0 && !sm.abort_flag) {
            record_error(p.status, kDevTimeoutFull);
            sm.abort_flag = 1u;
          }
          if (named_bar_red_or(kBarStage0 + slot, kHandoffThreads, !ok)) {
            stop = true;
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    constexpr int kHalf = 128;                 // columns per warp
    const uint32_t q = warp & 3u;              // TMEM lane quarter this warp may access
    const uint32_t ch = (warp - 2u) >> 2;      // which half of the 256 columns
    const uint32_t row = 32u * q + lane;
    const uint32_t et = threadIdx.x - 64u;     // 0..255
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    const uint32_t lead_acc_empty = mapa_shared(smem_u32(&sm.acc_empty), 0);
    if (fused) {
      // s and T of this CTA's 128 rows of each of its tiles, each 32-row slice
      // combined once per call
      const bool rows_ok = ensure_rows_of_tiles(p, sm, et, ntm2, ntn, cluster_id, nclusters, ntiles, rank);
      if (et == 0 && !rows_ok && !sm.abort_flag) {
        record_error(p.status, kDevTimeoutFinalize);
        sm.abort_flag = 1u;
      }
      if (et == 0 && lora) mbar_arrive(&sm.rows_ready);  // the producer may load T
    }
    int acc_count = 0;
    uint32_t g_fused = 0;  // FUSED: the stage counter of the compression
    for (int tile = cluster_id; tile < ntiles; tile += nclusters, ++acc_count) {
      if (FUSED) {
        const bool ok = compress_tile_stages<C>(sm, g_fused, nk, steps, et, lane);
        if (named_bar_red_or(kBarEpilogue, kEpiThreads, !ok)) {
          if (et == 0 && !sm.abort_flag) {
            record_error(p.status, kDevTimeoutFull);
            sm.abort_flag = 1u;
          }
          break;
        }
      }
      int pm, nb;
      pair_tile_coords(tile, ntm2, ntn, p.group_m, pm, nb);
      const int64_t grow = static_cast<int64_t>(pm) * 256 + rank * 128 + row;
      const bool row_ok = grow < p.M;
      const int64_t n_base = static_cast<int64_t>(nb) * 256;
      named_bar_sync(kBarEpilogue, kEpiThreads);  // the previous tile's bias is no longer read
      {
        const int64_t n = n_base + et;
        sm.bias_s[et] = (bias != nullptr && n < p.N) ? __bfloat162float(bias[n]) : 0.f;
      }
      // s of the row: with the fused combining step, written by the row block's
      // owner before the checks above (read past L1)
      float s = 1.f;
      if (row_ok) {
        if (p.fin_mode == 1) s = __ldcg(p.fin_scale + grow);
        else if (p.row_scale != nullptr) s = p.row_scale[grow];
      }
      bool ok = !sm.abort_flag;
      if (ok && !mbar_wait(&sm.acc_full, static_cast<uint32_t>(acc_count) & 1u)) {
        record_error(p.status, kDevTimeoutAccum);
        sm.abort_flag = 1u;
        ok = false;
      }
      if (named_bar_red_or(kBarEpilogue, kEpiThreads, !ok)) break;
      tc_fence_after();
      // The warp's 32 rows x 128 columns of the accumulator go to registers
      // first and the accumulator is handed back at once, so the next tile's
      // MMAs start while this tile is converted and stored: act(s * acc + bias)
      // -> bf16 -> 16-column pieces staged in shared memory -> asynchronous bulk
      // tensor stores (rows past M / columns past N are clipped by the TMA)
      const int32_t store_row = static_cast<int32_t>(pm * 256 + rank * 128 + 32 * q);
      uint8_t* my_stage = sm.ystage[warp - 2][0];
      uint32_t r[kHalf / 32][32];
#pragma unroll
      for (int c = 0; c < kHalf / 32; ++c)
        tmem_ld_32x32b_x32(sm.tmem_base + ((32u * q) << 16) + ch * kHalf + 32u * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
      int piece = 0;
#pragma unroll
      for (int c = 0; c < kHalf / 32; ++c) {
        const int col = static_cast<int>(ch) * kHalf + 32 * c;
#pragma unroll
        for (int h = 0; h < 2; ++h, ++piece) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int e = 16 * h + 2 * i;
            const float a = apply_act<ACT>(__fmaf_rn(s, __uint_as_float(r[c][e]), sm.bias_s[col + e]));
            const float b =
                apply_act<ACT>(__fmaf_rn(s, __uint_as_float(r[c][e + 1]), sm.bias_s[col + e + 1]));
            __nv_bfloat162 hv = __floats2bfloat162_rn(a, b);
            pk[i] = *reinterpret_cast<uint32_t*>(&hv);
          }
          uint8_t* buf = my_stage + 1024 * (piece & 1);
          if (lane == 0) bulk_wait_read_le1();  // the store that last used `buf` has read it
          __syncwarp();
          // row `lane`, 16-byte chunks k = 0,1 at 32B-swizzled positions
          const uint32_t sw = (lane >> 2) & 1u;
          *reinterpret_cast<uint4*>(buf + lane * 32 + ((0u ^ sw) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(buf + lane * 32 + ((1u ^ sw) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tm_y, buf, static_cast<int32_t>(n_base + col + 16 * h), store_row);
            bulk_commit();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // every Y tile this warp issued is written
  }

  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, copies and epilogues are all finished
  if (warp == 1) tmem_dealloc_pair(sm.tmem_base, kTmemCols);
}

// the opt-in limit of dynamic shared memory per block on sm_100 (227 KB), with
// the 1 KB the kernel spends on aligning its base
static_assert(sizeof(PairSmem<true, false>) + 1024 <= 232448, "sparse pair GEMM shared memory");
static_assert(sizeof(PairSmem<false, false>) + 1024 <= 232448, "dense pair GEMM shared memory");
static_assert(sizeof(PairSmem<true, true>) + 1024 <= 232448, "fused pair GEMM shared memory");

template <bool SPARSE, int ACT, bool FUSED>
cudaError_t configure_pair_variant() {
  static std::once_flag once[64];
  static cudaError_t configured[64];
  return once_per_device(once, configured, []() {
    return cudaFuncSetAttribute(lynx_gemm_pair_kernel<SPARSE, ACT, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(PairSmem<SPARSE, FUSED>) + 1024));
  });
}

template <bool SPARSE, int ACT, bool FUSED>
cudaLaunchConfig_t pair_config(int grid, cudaStream_t stream, cudaLaunchAttribute (&attr)[2]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(PairSmem<SPARSE, FUSED>) + 1024;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <bool SPARSE, int ACT, bool FUSED>
cudaError_t launch_pair_variant(const GemmLaunch& p, cudaStream_t stream) {
  cudaError_t e = configure_pair_variant<SPARSE, ACT, FUSED>();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<SPARSE, ACT, FUSED>(p.grid, stream, attr);
  return cudaLaunchKernelEx(&cfg, lynx_gemm_pair_kernel<SPARSE, ACT, FUSED>, p);
}

template <bool SPARSE, int ACT, bool FUSED>
int pair_max_clusters_variant() {
  static std::once_flag once[64];
  static int clusters[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::call_once(once[dev], [dev]() {
    clusters[dev] = 0;
    if (configure_pair_variant<SPARSE, ACT, FUSED>() != cudaSuccess) return;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pair_config<SPARSE, ACT, FUSED>(2, nullptr, attr);
    cfg.numAttrs = 1;  // the cluster shape is what matters here
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lynx_gemm_pair_kernel<SPARSE, ACT, FUSED>, &cfg) == cudaSuccess)
      clusters[dev] = n;
    else
      (void)cudaGetLastError();  // a failed query is not sticky; the caller falls back
  });
  return clusters[dev];
}

}  // namespace

int gemm_pair_max_clusters(bool sparse, int act, bool fused) {
  if (fused)
    return act == kActGeluTanh ? pair_max_clusters_variant<true, kActGeluTanh, true>()
                               : pair_max_clusters_variant<true, kActNone, true>();
  if (act == kActGeluTanh)
    return sparse ? pair_max_clusters_variant<true, kActGeluTanh, false>()
                  : pair_max_clusters_variant<false, kActGeluTanh, false>();
  return sparse ? pair_max_clusters_variant<true, kActNone, false>() : pair_max_clusters_variant<false, kActNone, false>();
}

cudaError_t launch_gemm_pair(const GemmLaunch& p, cudaStream_t stream) {
  if (p.fused)
    return p.act == kActGeluTanh ? launch_pair_variant<true, kActGeluTanh, true>(p, stream)
                                 : launch_pair_variant<true, kActNone, true>(p, stream);
  if (p.act == kActGeluTanh)
    return p.sparse ? launch_pair_variant<true, kActGeluTanh, false>(p, stream)
                    : launch_pair_variant<false, kActGeluTanh, false>(p, stream);
  return p.sparse ? launch_pair_variant<true, kActNone, false>(p, stream)
                  : launch_pair_variant<false, kActNone, false>(p, stream);
}

}  // namespace lynx
