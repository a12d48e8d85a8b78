// Block-scaled MXFP4 GEMM on CTA pairs (tcgen05 cta_group::2): the same Y = Xq . Wq^T as
// bat_gemm.cuh (BATQuant note, en.papernotes.org, Method > Key Designs 1: the low-bit
// product Q(XP) . Q(P^-1 W^T)), for shapes with more than one 128-row tile.
//
// Why pairs. A 256 x 256 tile on a cluster of two CTAs: each CTA loads its own 128 rows
// of X and half (128 rows) of the tile's 256 W rows, and one M=256 MMA issued by the even
// CTA reads A and B from both CTAs' shared memory and writes each CTA's 128 rows of the
// accumulator in its own TMEM. Per SM and k-step the copies shrink from 48 KB of codes
// (one-SM kernel, 128 x 256 tile) to 32 KB (plus 3 KB of scales), the L2 reads of W
// halve, and six stages fit in shared memory instead of four.
//
// Synchronisation (barriers at the same offsets in both CTAs):
//   code tiles: both CTAs' tensor copies of a stage complete on the even CTA's full
//     barrier (cta_group::2 copies may signal the peer's barrier); the even CTA's
//     producer expects the bytes of all four copies;
//   scales: each CTA loads its 128 rows' X scales and the W scales of all 256 rows into
//     its own stage (local sf_full barrier) and its writer warps store them into its own
//     TMEM (each CTA's TMEM must hold the scales of all 256 W rows), then arrive on the
//     even CTA's sf_ready barrier: the even CTA's writers after also waiting for the
//     stage's full barrier, so that sf_ready alone tells the issuers that the stage is
//     ready; the odd CTA's writers with a relaxed remote arrival (see mbar_arrive_remote);
//   two MMA issuer threads in the even CTA take alternate k-steps in a fixed order, issue
//     the stage's MMAs and commit to both CTAs' empty barriers (multicast commit); after a
//     tile each commits to both CTAs' tmem_full;
//   each CTA's epilogue drains its own TMEM rows and arrives on the even CTA's
//     tmem_empty.
// No copy is multicast. Every wait is bounded and reports through the error word; both
// CTAs meet at a cluster barrier before TMEM is released.
//
// Tile-level overlap with the prologue (p.cta_flags set): instead of waiting for the
// prologue's grid to retire, the code producer warp's lanes 1-31 walk this CTA's tiles
// ahead of the producers and, for each, poll the completion flags of the prologue CTAs
// that wrote the 128-row token tile this CTA loads (in every strip, the one or two CTAs
// whose unit range covers the tile), then publish "tiles ready" in shared memory; the
// code and scale producers wait for that count before a tile's first X copy.
// The weights and their scales are not written by the prologue, and neither is Y.
//
// Warp roles per CTA: 0-3 epilogue, 4-7 scale writers, 8 code producer, 9 MMA issuer of
// even k-steps (even CTA) / TMEM owner (both), 10 scale producer, 11 MMA issuer of odd
// k-steps (even CTA).
#pragma once

#include "bat_common.cuh"
#include "bat_gemm.cuh"

namespace bat {

namespace gemm2 {
constexpr int kRows = 128;                    // rows of X per CTA (the pair's tile is 256)
constexpr int kBN = 256;                      // rows of W per tile (MMA N), 128 per CTA
constexpr int kBK = 256;                      // K elements per stage (128 bytes of codes per row)
constexpr int kStages = 6;
constexpr int kABytes = kRows * 128;          // 16 KB
constexpr int kBBytes = (kBN / 2) * 128;      // 16 KB: this CTA's half of the W tile
constexpr int kChunk = 512;                   // 128 rows x 4 scale bytes
constexpr int kSfaBytes = 2 * kChunk;         // this CTA's 128 rows, two 128-K chunks
constexpr int kSfbBytes = 2 * 2 * kChunk;     // all 256 W rows (two groups), two chunks
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 35 KB
static_assert(kStageBytes % 1024 == 0, "stage alignment for the 128-byte swizzle");
constexpr int kThreads = 384;
// bf16 output staging for the TMA store: 128 rows x 32 columns (64 bytes, 64-byte swizzle)
constexpr int kEpiBytes = kRows * 64;
constexpr int kSmemBytes = kStages * kStageBytes + kEpiBytes + 1024 /*align*/ + 512 /*barriers*/;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr uint32_t kRegsEpi = gemm::kRegsEpi;
constexpr uint32_t kRegsOther = gemm::kRegsOther;
// TMEM (both CTAs): accumulator [0, 256); stage s's scales at 256 + 24 s: A words [0, 8)
// (two chunks x 4), B words [8, 24) (two chunks x two 128-row groups x 4)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;
constexpr uint32_t kSfStageCols = 24;
static_assert(kSfCol0 + kStages * kSfStageCols <= kTmemCols, "TMEM columns");
}  // namespace gemm2

// ---------------------------------------------------------------- pair helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of this CTA's shared-memory address `a` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// Arrival on a barrier of either CTA of the pair, relaxed. Both signals sent this way
// hand over tensor memory only: the scale writers' tcgen05.st (scales ready) and the
// epilogue's tcgen05.ld (accumulator free). The sender has waited for those operations to
// complete (tcgen05.wait::st / wait::ld) and ordered them before the arrival with
// tcgen05.fence::before_thread_sync; the receiver waits with acquire and orders its MMAs
// after with tcgen05.fence::after_thread_sync. No generic-memory data rides on these
// arrivals. Timed in this kernel, a release arrival at cluster scope held its thread for
// about 650 ns, which made the scale hand-off the bound of the k-loop; the relaxed form
// takes about 10 ns.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// mbar_wait with acquire at cluster scope: for phases completed by the peer CTA's
// release arrivals (or its copies).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_cluster_now(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, unsigned int code) {
  if (mbar_try_wait_cluster_now(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity, 100000u)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_dev_error, code);
      return false;
    }
  }
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Tensor copy into this CTA's shared memory whose completion is counted on a barrier that
// may be in the peer CTA of the pair (`bar` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive (once the issuing thread's earlier MMAs are done) on the barrier at this address
// in every CTA of `mask` (bit r: CTA rank r of the pair).
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// D (+)= (A * 2^sfa) x (B * 2^sfb)^T on the pair: M = 256 (128 rows per CTA), K = 64.
__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// tmap_a: Xq codes, box 128 bytes x 128 rows; tmap_b: Wq codes, box 128 bytes x 128 rows
// (each CTA its half of the W tile); tmap_y: bf16 Y, box 32 columns x 128 rows, 64-byte
// swizzle (used when p.tma_store). p.splits is unused (always 1).
__global__ void __launch_bounds__(gemm2::kThreads, 1)
    bat_mxf4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                              const __grid_constant__ CUtensorMap tmap_b,
                              const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  using namespace gemm2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  // stage s: [A 16K][B 16K][SFA 1K][SFB 2K]; then the epilogue staging; then barriers
  const uint32_t stg = base + kStages * kStageBytes;
  const uint32_t bars = stg + kEpiBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };                   // used in CTA 0
  auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };      // both
  auto sf_full = [&](int s) { return bars + 8u * (2 * kStages + s); };    // both (local)
  auto sf_ready = [&](int s) { return bars + 8u * (3 * kStages + s); };   // used in CTA 0
  const uint32_t tmem_full = bars + 8u * (4 * kStages);                   // both
  const uint32_t tmem_empty = tmem_full + 8u;                             // used in CTA 0
  const uint32_t turn_bar = tmem_empty + 8u;                             // used in CTA 0
  const uint32_t tiles_ready = turn_bar + 8u;  // tile-level overlap: tiles whose X is written
  const uint32_t tmem_slot = tiles_ready + 8u;
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(base_ptr + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0: issues the MMAs; 1: its peer
  const bool even = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);     // CTA 0's producer arrival (+ both CTAs' copy bytes)
      mbar_init(empty_bar(s), 1);    // the multicast commit
      mbar_init(sf_full(s), 1);      // this CTA's scale producer (+ its scale copy bytes)
      mbar_init(sf_ready(s), 8);     // four writer warps in each CTA
    }
    mbar_init(tmem_full, 2);         // the multicast commits of the two issuers
    mbar_init(turn_bar, 1);          // the issuer of the k-step just issued
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(tiles_ready), "r"(0u) : "memory");
    mbar_init(tmem_empty, 8);        // four epilogue warps in each CTA
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (p.tma_store) prefetch_tmap(&tmap_y);
  }
  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  // Everything above is local setup; the operands (and Y) belong to the kernels before
  // (with p.cta_flags, X and its scales are waited for tile by tile below instead).
  if (p.cta_flags == nullptr) grid_dependency_wait();

  const int64_t m_tiles = (p.M + 2 * kRows - 1) / (2 * kRows);  // 256-row tiles
  const int64_t n_tiles = (p.N + kBN - 1) / kBN;
  const int64_t tiles = m_tiles * n_tiles;
  const int k_stages = static_cast<int>((p.K + kBK - 1) / kBK);
  const int64_t pair_id = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;
  const int64_t sf_groups_a = (p.M + 127) / 128;  // 128-row groups of the X scale layout
  const int64_t sf_groups_b = (p.N + 127) / 128;
  bool ok = true;

  // (tile-level overlap) the producers' wait for the i-th tile of this CTA's walk
  auto wait_tile_ready = [&](uint32_t i) -> bool {
    if (p.cta_flags == nullptr) return true;
    if (ld_acquire_cta_u32(tiles_ready) <= i) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_cta_u32(tiles_ready) <= i) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          atomicOr(&g_dev_error, kErrWaitFull);
          return false;
        }
        __nanosleep(64);
      }
    }
    // (the prologue's threads made their writes visible to the async proxy, which the
    // copies read through, before publishing them)
    return true;
  };

  if (warp >= 8) setmaxnreg_dec<kRegsOther>();  // warpgroup 2
  if (warp == 8) {
    // ------------------------------------------------------------ code producer (both)
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(full_bar(0), 0);  // CTA 0's full barriers
      int stage = 0;
      uint32_t phase = 0;
      uint32_t inflight = 0;  // bit s: stage s was loaded; bit 16+s: parity of that load
      uint32_t ti = 0;  // tiles of this CTA's walk so far
      for (int64_t tile = pair_id; tile < tiles && ok; tile += npairs, ++ti) {
        const int64_t mt = tile % m_tiles;
        const int64_t nt = tile / m_tiles;
        const int32_t arow = static_cast<int32_t>(mt * 2 * kRows + kRows * rank);
        const int32_t brow = static_cast<int32_t>(nt * kBN + (kBN / 2) * rank);
        if (!wait_tile_ready(ti)) { ok = false; break; }
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          // both CTAs' copies land on CTA 0's barrier, which expects all four (rows past
          // the ends are zero-filled and still counted)
          if (even) mbar_expect_tx(full_bar(stage), 2u * (kABytes + kBBytes));
          const uint32_t sa = base + stage * kStageBytes;
          tma_load_2d_pair(sa, &tmap_a, full0 + 8u * stage, ks * 128, arow);
          tma_load_2d_pair(sa + kABytes, &tmap_b, full0 + 8u * stage, ks * 128, brow);
          inflight = (inflight & ~(0x10001u << stage)) | (1u << stage) | (phase << (16 + stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // CTA 0 drains the stages (its barrier counts both CTAs' copies); CTA 1's copies are
      // covered by CTA 0's drain and the cluster barrier before exit
      if (even)
        for (int s = 0; s < kStages; ++s)
          if ((inflight >> s) & 1u) mbar_wait_cluster(full_bar(s), (inflight >> (16 + s)) & 1u, kErrWaitFull);
    } else if (p.cta_flags != nullptr) {
      // lanes 1-31: the flags of each tile's token tile, ahead of the producers. Relaxed
      // polls, then an acquire fence once all are seen; lane 1 then counts the tile ready
      // (release, CTA scope) for the producers.
      const unsigned mask = 0xfffffffeu;
      uint32_t ti = 0;
      for (int64_t tile = pair_id; tile < tiles; tile += npairs, ++ti) {
        const int64_t t = (tile % m_tiles) * 2 + rank;  // this CTA's 128-row token tile
        if (t < p.q_mtiles) {
          const uint64_t t0 = globaltimer_ns();
          bool stalled = false;
          while (true) {
            bool mine = true;
            for (int st = lane - 1; st < p.q_strips; st += 31) {
              // strip st: units v = tile * npair + pair, split over q_cps CTAs as
              // [sunits c / cps, sunits (c + 1) / cps); those holding units of token tile t
              const int64_t npair = min(4, p.q_nbp2 - 4 * st);
              const int64_t sunits = p.q_mtiles * npair;
              const int64_t u0 = t * npair, u1 = (t + 1) * npair - 1;
              int64_t c = u0 * p.q_cps / sunits;
              while (c > 0 && sunits * c / p.q_cps > u0) --c;
              while (c + 1 < p.q_cps && sunits * (c + 1) / p.q_cps <= u0) ++c;
              for (; c < p.q_cps && sunits * c / p.q_cps <= u1; ++c) {
                unsigned long long v;
                asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];"
                             : "=l"(v)
                             : "l"(p.cta_flags + st * p.q_cps + c)
                             : "memory");
                mine = mine && v == p.q_epoch;
              }
            }
            if (__all_sync(mask, mine)) break;
            // (a warp-wide decision: every lane leaves the loop together)
            if (__any_sync(mask, globaltimer_ns() - t0 > kWaitLimitNs)) { stalled = true; break; }
            __nanosleep(128);
          }
          if (stalled) {
            if (lane == 1) atomicOr(&g_dev_error, kErrWaitFull);
            break;
          }
          asm volatile("fence.acq_rel.gpu;" ::: "memory");
        }
        __syncwarp(mask);
        if (lane == 1) asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(tiles_ready), "r"(ti + 1)
                                    : "memory");
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ scale producer (both)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t inflight = 0;
      uint32_t ti = 0;
      for (int64_t tile = pair_id; tile < tiles && ok; tile += npairs, ++ti) {
        const int64_t mt = tile % m_tiles;
        const int64_t nt = tile / m_tiles;
        const int64_t ga = mt * 2 + rank;                        // this CTA's X row group
        if (!wait_tile_ready(ti)) { ok = false; break; }
        const bool has_a = ga < sf_groups_a;                     // rows past M: no scales
        const int ngb = (nt * 2 + 1 < sf_groups_b) ? 2 : 1;      // W row groups of the tile
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          const int c0 = ks * 2;
          const int nch = min(2, p.nbp4 - c0);
          const uint32_t bytes = static_cast<uint32_t>(nch) * kChunk * ((has_a ? 1 : 0) + ngb);
          const uint32_t sa = base + stage * kStageBytes + kABytes + kBBytes;
          mbar_expect_tx(sf_full(stage), bytes);
          if (has_a) bulk_load(sa, p.sfa + (ga * p.nbp4 + c0) * kChunk, nch * kChunk, sf_full(stage));
          for (int g = 0; g < ngb; ++g)
            bulk_load(sa + kSfaBytes + g * (2 * kChunk), p.sfb + ((nt * 2 + g) * p.nbp4 + c0) * kChunk,
                      nch * kChunk, sf_full(stage));
          inflight = (inflight & ~(0x10001u << stage)) | (1u << stage) | (phase << (16 + stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < kStages; ++s)
        if ((inflight >> s) & 1u) mbar_wait(sf_full(s), (inflight >> (16 + s)) & 1u, kErrWaitFull);
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------ MMA issuers (CTA 0)
    // Warp 9 issues the even k-steps of this CTA's walk, warp 11 the odd ones; each waits
    // for the other's previous k-step to be issued (turn barrier), so the MMAs enter the
    // tensor pipe in k order and the sums are the same as from one thread. Each thread
    // commits its own k-steps' stages and, at the end of every tile, tmem_full (count 2).
    if (lane == 0 && even) {
      const uint32_t iss = warp == 9 ? 0u : 1u;
      // Descriptors of stage 0; other stages and K sub-blocks only move the start
      // address field (16-byte units). The same offsets address both CTAs' tiles.
      const uint64_t adesc0 = smem_desc(base, 16, 1024, 2);
      const uint64_t bdesc0 = smem_desc(base + kABytes, 16, 1024, 2);
      constexpr uint32_t kStageU = kStageBytes >> 4;
      const uint32_t id_lo = idesc_mxf4(2 * kRows, kBN, 0, 0);
      const uint32_t id_hi = idesc_mxf4(2 * kRows, kBN, 2, 2);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      uint32_t g = 0;
      for (int64_t tile = pair_id; tile < tiles && ok; tile += npairs) {
        for (int ks = 0; ks < k_stages; ++ks, ++g) {
          if ((g & 1u) == iss) {
            if (ks == 0 && !mbar_wait_cluster(tmem_empty, acc_phase ^ 1u, kErrWaitTmemEmpty)) { ok = false; break; }
            if (g > 0 && !mbar_wait(turn_bar, (g - 1u) & 1u, kErrWaitFull)) { ok = false; break; }
            
            // scales of both CTAs in TMEM; the even CTA's writers arrive only once the
            // stage's code copies have landed, so this one wait covers the codes too
            if (!mbar_wait_cluster(sf_ready(stage), phase, kErrWaitFull)) { ok = false; break; }
            tc_fence_after();
            const uint64_t so = static_cast<uint64_t>(stage) * kStageU;
            const uint32_t t_sfa = tmem_base + kSfCol0 + kSfStageCols * stage;
            const uint32_t t_sfb = t_sfa + 8;
            const int64_t krem = p.K - static_cast<int64_t>(ks) * kBK;
            const uint32_t acc0 = ks != 0 ? 1u : 0u;
            if (krem >= kBK) {
              mma_mxf4_pair(tmem_base, adesc0 + so, bdesc0 + so, id_lo, t_sfa, t_sfb, acc0);
              mma_mxf4_pair(tmem_base, adesc0 + so + 2, bdesc0 + so + 2, id_hi, t_sfa | (2u << 30),
                            t_sfb | (2u << 30), 1u);
              mma_mxf4_pair(tmem_base, adesc0 + so + 4, bdesc0 + so + 4, id_lo, t_sfa + 4, t_sfb + 8, 1u);
              mma_mxf4_pair(tmem_base, adesc0 + so + 6, bdesc0 + so + 6, id_hi, (t_sfa + 4) | (2u << 30),
                            (t_sfb + 8) | (2u << 30), 1u);
            } else {
              const int nkb = static_cast<int>((krem + 63) / 64);
              for (int kq = 0; kq < nkb; ++kq) {
                const uint32_t hi = static_cast<uint32_t>(kq & 1);
                const uint32_t c = static_cast<uint32_t>(kq >> 1);
                mma_mxf4_pair(tmem_base, adesc0 + so + 2 * kq, bdesc0 + so + 2 * kq, hi ? id_hi : id_lo,
                              (t_sfa + 4 * c) | (hi << 31), (t_sfb + 8 * c) | (hi << 31),
                              (acc0 | static_cast<uint32_t>(kq)) != 0 ? 1u : 0u);
              }
            }
            tc_commit_pair(empty_bar(stage), 0x3);  // both CTAs may refill this stage
            mbar_arrive(turn_bar);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        tc_commit_pair(tmem_full, 0x3);  // both CTAs' accumulator rows (once per issuer)
        acc_phase ^= 1u;
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ scale-factor writers
    setmaxnreg_dec<kRegsOther>();
    // Warp w writes TMEM lane quarter q = w % 4 of this CTA: lane l holds TMEM lane 32q + l,
    // which takes 16-byte row l of every 512-byte chunk at the chunk's four words.
    const int q = warp & 3;
    const uint32_t tlane = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t ready0 = mapa_shared(sf_ready(0), 0);
    int stage = 0;
    uint32_t phase = 0;
    for (int64_t tile = pair_id; tile < tiles && ok; tile += npairs) {
      for (int ks = 0; ks < k_stages; ++ks) {
        if (!mbar_wait(sf_full(stage), phase, kErrWaitFull)) { ok = false; break; }
        if (even && !mbar_wait_cluster(full_bar(stage), phase, kErrWaitFull)) { ok = false; break; }
        const uint32_t ssf = base + stage * kStageBytes + kABytes + kBBytes + lane * 16;
        uint32_t fa[8], fb[16];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 v = lds_v4_u32(ssf + c * kChunk);
          fa[4 * c] = v.x; fa[4 * c + 1] = v.y; fa[4 * c + 2] = v.z; fa[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const uint4 v = lds_v4_u32(ssf + kSfaBytes + g * (2 * kChunk) + c * kChunk);
            const int w = 8 * c + 4 * g;
            fb[w] = v.x; fb[w + 1] = v.y; fb[w + 2] = v.z; fb[w + 3] = v.w;
          }
        const uint32_t tcol = tmem_base + tlane + kSfCol0 + kSfStageCols * stage;
        tmem_st_32x32b_x8(tcol, fa);
        tmem_st_32x32b_x16(tcol + 8, fb);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (even) mbar_arrive(sf_ready(stage));  // release (CTA scope): covers the code copies
          else mbar_arrive_remote(ready0 + 8u * stage);
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue (both)
    setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;
    const int rl = 32 * q + lane;  // row within this CTA's 128 rows
    const bool leader = (warp == 0 && lane == 0);
    const uint32_t empty0 = mapa_shared(tmem_empty, 0);
    uint32_t acc_phase = 0;
    for (int64_t tile = pair_id; tile < tiles && ok; tile += npairs) {
      const int64_t mt = tile % m_tiles;
      const int64_t nt = tile / m_tiles;
      const int64_t row0 = mt * 2 * kRows + kRows * rank;  // first row of this CTA's rows
      bool got = mbar_wait_cluster(tmem_full, acc_phase, kErrWaitTmemFull);
      if (p.tma_store) got = epi_bar_and(got);
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      if (p.tma_store) {
        // 1) drain the accumulator into registers as bf16 pairs and release TMEM at once
        //    (four 32-column loads per wait: two round trips instead of eight)
        uint32_t h[kBN / 2];
#pragma unroll
        for (int hh = 0; hh < kBN / 128; ++hh) {
          uint32_t r[4][32];
#pragma unroll
          for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(trow + (hh * 4 + i) * 32, r[i]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[i][2 * c]), __uint_as_float(r[i][2 * c + 1]));
              h[(hh * 4 + i) * 16 + c] = *reinterpret_cast<uint32_t*>(&v);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(empty0);  // accumulator free: next tile's MMAs may start
        // 2) stream 32-column slices through the staging box; 16-byte chunk j of row rl sits
        //    at chunk (j ^ ((rl / 2) % 4)) (the 64-byte swizzle of the store's tensor map)
        const uint32_t rowb = stg + rl * 64;
#pragma unroll
        for (int b = 0; b < kBN / 32; ++b) {
          if (leader) bulk_wait_read0();  // the previous slice has left the box
          epi_bar_sync();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(rowb + ((j ^ ((rl >> 1) & 3)) << 4), h[b * 16 + 4 * j], h[b * 16 + 4 * j + 1],
                         h[b * 16 + 4 * j + 2], h[b * 16 + 4 * j + 3]);
          fence_async_smem();
          epi_bar_sync();
          const int64_t col = nt * kBN + 32 * b;
          if (leader && col < p.N && row0 < p.M) {
            tma_store_2d(&tmap_y, stg, static_cast<int32_t>(col), static_cast<int32_t>(row0));
            bulk_commit();
          }
        }
      } else {
        const int64_t row = row0 + rl;
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + cc * 32, r);
          tmem_wait_ld();
          store_chunk(p, row, nt * kBN + cc * 32, r);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(empty0);
      }
      acc_phase ^= 1u;
    }
    if (leader) bulk_wait0();
  }

  // both CTAs stay until every remote arrival and every MMA reading their shared memory is
  // done; CTA 0 waits for its last MMAs through the final tmem_full commit seen by its
  // epilogue (or, on an error path, the bounded waits above)
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 9) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace bat
