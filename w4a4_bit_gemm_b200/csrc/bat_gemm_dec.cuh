// Decode-shaped MXFP4 GEMM (at most 64 activation rows): the same Y = Xq . Wq^T as
// bat_gemm.cuh (BATQuant note, en.papernotes.org, Method > Key Designs 1: the low-bit
// product Q(XP) . Q(P^-1 W^T)), computed as its transpose Y^T = Wq . Xq^T.
//
// With a handful of tokens the GEMM streams the weights once and does almost no
// arithmetic. The 128-lane MMA dimension therefore runs over weight rows (M = 128 W
// rows per tile) and the tokens become the MMA's N (16 to 64, zero rows past M), so no
// MMA lane computes a padding row. The W tiles are split along K over a cluster of S
// CTAs; rank r takes K stages [r ks / S, (r+1) ks / S), at most kStages of them, so
// every stage has its own shared-memory slot and all copies are in flight at once.
//
// Each TMA or tcgen05 instruction holds its issuing thread for some 60-80 ns, which at
// these sizes is what bounds the kernel, so the per-stage instruction count is kept to
// one W tensor copy (producer) and four MMAs, and the stages alternate between two
// issuer threads with an accumulator each (even stages into the first, odd into the
// second; the epilogue adds the two, first + second, a fixed order). The rest goes
// through the four epilogue warps, idle until the accumulators are ready:
//   - the scales of W and X come straight from global memory into registers and are
//     stored into TMEM (tcgen05.st) in the layout the block-scaled MMA reads, all stages
//     at once;
//   - the X codes of all stages (a few KB) are read with plain loads and stored into
//     shared memory in the 128-byte-swizzled layout of a tensor copy, zeros past M and K.
// They then arrive on one barrier, which the issuer waits for once.
//
// Programmatic stream serialization: the kernel may start while the kernel before it
// finishes. Xq, its scales and Y are only touched after griddepcontrol.wait, or, inside
// a linear layer, after the row quantizer's completion flags (q_flags): each of its q_ctas
// CTAs stores this call's epoch there with release semantics once its outputs are
// written, and the four epilogue warps wait (acquire, bounded) for all of them; the grid
// dependency would wait for the whole quantizer grid to retire. That kernel never writes
// the weights, and the layer says so (w_static): the weight copies and the weight scales
// then start at once.
// Otherwise the producer only prefetches the W boxes into L2 (the point of coherence, so
// a later write would still be seen) before waiting.
//
// Split-K sum: rows [o 128 / S, (o+1) 128 / S) of the tile belong to rank o. Every other
// rank sends its fp32 partial of such a row (the row's token values, contiguous) into
// rank o's shared memory with st.async, which counts the bytes on rank o's receive
// barrier; the thread of rank o that holds the row's own partial puts it beside them,
// waits for that barrier, adds the S partials in rank order (a fixed order, so the result
// does not depend on timing) and stages the row for the write-out; no cluster barrier
// follows the sends. Every wait is bounded and reports through the error word; every CTA
// takes part in the one cluster barrier phase (all CTAs started), error or not.
#pragma once

#include "bat_common.cuh"
#include "bat_gemm.cuh"

namespace bat {

namespace gemmd {
constexpr int kBM = 128;                      // W rows per tile (MMA M)
constexpr int kBK = 256;                      // K elements per stage (128 bytes of codes per row)
constexpr int kMaxNx = 64;                    // token rows per MMA (N), a multiple of 16
constexpr int kStages = 8;                    // stage slots = K stages per CTA at most
constexpr int kWBytes = kBM * 128;            // 16 KB per stage
constexpr int kXBytes = kMaxNx * 128;         // 8 KB per stage at most (nx * 128 used)
constexpr int kRedBytes = kMaxNx * kBM * 4;   // pushed partials: [rank][owned row][64 tokens]
constexpr int kThreads = 224;                 // warps 0-3 epilogue, 4 producer, 5-6 issuers
constexpr int kSmemBytes = kStages * (kWBytes + kXBytes) + kRedBytes + 1024 /*align*/ + 256;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr int kChunk = 512;                   // one 128-K chunk of scales of 128 rows
// TMEM: accumulators [0, 64) (even stages) and [64, 128) (odd stages); stage s's scales at
// 128 + 16 s: W chunk words [0, 8), X [8, 16)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kAccCols = 64;
constexpr uint32_t kSfCol0 = 128;
constexpr uint32_t kSfStageCols = 16;
static_assert(kSfCol0 + kStages * kSfStageCols <= kTmemCols, "TMEM columns");
constexpr int kMaxSplits = 8;
}  // namespace gemmd

// Explicit state-space accesses for the epilogue. (In this cluster kernel a generic
// load or store of shared or global memory was timed at some 200-300 ns per access in
// the epilogue's dependent chains; the shared::cta / shared::cluster / global forms are
// not.)
__device__ __forceinline__ void sts_b16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ void sts_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void stg_v4(void* ptr, uint4 v) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void stg_b16(void* ptr, uint16_t v) {
  asm volatile("st.global.b16 [%0], %1;" ::"l"(ptr), "h"(v) : "memory");
}
__device__ __forceinline__ void stg_b32(void* ptr, uint32_t v) {
  asm volatile("st.global.b32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
// (The received rows are 256 bytes apart; 16-byte chunk c of row r sits at slot c ^ (r % 8)
// of its row, so that the owner threads of eight consecutive rows read different banks.)
// 16 bytes into the shared memory of CTA `rank` of the cluster at this CTA's offset
// `addr`, counted (complete_tx) on the barrier at offset `bar` in that CTA
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint32_t bar, uint32_t rank, uint4 v) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(addr), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(bar), "r"(rank));
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(ra),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(rb)
      : "memory");
}

// Prefetch a box of a 2-D tensor map into L2 (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// tmap_w: Wq codes, box 128 bytes x 128 rows, 128-byte swizzle. nx = M rounded up to 16
// (<= 64). p.splits = S, the cluster size: 1, 2, 4 or 8; the grid is ceil(N / 128) x S
// CTAs and ceil(ceil(K / 256) / S) <= kStages. w_static != 0: the kernel before does not
// write the weights or their scales. q_flags: null (wait for the grid dependency) or the
// row quantizer's q_ctas completion flags, complete when all hold `epoch`.
__global__ void __launch_bounds__(gemmd::kThreads, 1)
    bat_mxf4_gemm_dec_kernel(const __grid_constant__ CUtensorMap tmap_w, const GemmParams p,
                             const uint8_t* __restrict__ xcodes, const int nx, const int w_static,
                             const unsigned long long* __restrict__ q_flags, const int q_ctas,
                             const unsigned long long epoch) {
  using namespace gemmd;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  // [W: kStages x 16 KB][X: kStages x nx x 128 B][partials][barriers]
  const uint32_t xbase = base + kStages * kWBytes;
  const uint32_t red = base + kStages * (kWBytes + kXBytes);  // shared address of the partials
  const uint32_t bars = base + kStages * (kWBytes + kXBytes) + kRedBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  const uint32_t ready_bar = bars + 8u * kStages;  // X codes in shared memory, scales in TMEM
  const uint32_t tmem_full = ready_bar + 8u;
  const uint32_t red_bar = tmem_full + 8u;  // the peers' partials of the owned rows
  const uint32_t tmem_slot = red_bar + 8u;
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(base_ptr + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.splits;
  const int rank = static_cast<int>(blockIdx.x % S);
  const int64_t tile = blockIdx.x / S;
  const int k_stages = static_cast<int>((p.K + kBK - 1) / kBK);
  const int kb = rank * k_stages / S;
  const int nk = (rank + 1) * k_stages / S - kb;  // 1 .. kStages
  const int32_t wrow = static_cast<int32_t>(tile * kBM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(full_bar(s), 1);
    mbar_init(ready_bar, 4);
    mbar_init(tmem_full, 2);  // one commit per issuer
    mbar_init(red_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // the bytes the S - 1 peers send: their partials of this rank's kBM / S rows
    if (S > 1) mbar_expect_tx(red_bar, static_cast<uint32_t>((S - 1) * (kBM / S) * nx * 4));
    prefetch_tmap(&tmap_w);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // Cluster barrier: every CTA has started and initialised its receive barrier before any
  // thread writes into a peer's shared memory (arrive now, wait right before sending; the
  // barrier initialisation fence above makes the arrival a release).
  if (S > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  // warps 0-3: the tile row rl (TMEM lane) whose accumulator values r[][] (tokens) they hold
  const int rl = 32 * warp + lane;
  uint32_t r[2][32] = {};
  bool got = false;

  if (warp == 4) {
    // ------------------------------------------------------------ producer: W tiles
    if (lane == 0) {
      if (!w_static) {
        for (int s = 0; s < nk; ++s) tma_prefetch_2d(&tmap_w, (kb + s) * 128, wrow);
        grid_dependency_wait();
      }
      for (int s = 0; s < nk; ++s) {
        mbar_expect_tx(full_bar(s), kWBytes);
        tma_load_2d(base + s * kWBytes, &tmap_w, full_bar(s), (kb + s) * 128, wrow);
      }
      // no copy may still be writing shared memory when the CTA moves on (bounded)
      for (int s = 0; s < nk; ++s) mbar_wait(full_bar(s), 0, kErrWaitFull);
    }
  } else if (warp == 5 || warp == 6) {
    // ------------------------------------------------------------ MMA issuers
    // warp 5 issues the even stages into accumulator 0, warp 6 the odd ones into 1
    if (lane == 0) {
      const int iss = warp - 5;
      const uint32_t acc = tmem_base + kAccCols * iss;
      const uint64_t wdesc0 = smem_desc(base, 16, 1024, 2);
      const uint64_t xdesc0 = smem_desc(xbase, 16, 1024, 2);
      const uint32_t id_lo = idesc_mxf4(kBM, nx, 0, 0);  // scale bytes 0-1 of each word
      const uint32_t id_hi = idesc_mxf4(kBM, nx, 2, 2);  // scale bytes 2-3
      if (mbar_wait(ready_bar, 0, kErrWaitFull)) {
        for (int s = iss; s < nk; s += 2) {
          if (!mbar_wait(full_bar(s), 0, kErrWaitFull)) break;
          tc_fence_after();
          // descriptor start addresses in 16-byte units
          const uint64_t wo = static_cast<uint64_t>(s) * (kWBytes >> 4);
          const uint64_t xo = static_cast<uint64_t>(s) * static_cast<uint64_t>(nx * 8);
          const uint32_t t_sfw = tmem_base + kSfCol0 + kSfStageCols * s;
          const uint32_t t_sfx = t_sfw + 8;
          const int64_t krem = p.K - static_cast<int64_t>(kb + s) * kBK;
          const int nkb = krem >= kBK ? 4 : static_cast<int>((krem + 63) / 64);
          for (int kq = 0; kq < nkb; ++kq) {
            const uint32_t hi = static_cast<uint32_t>(kq & 1);
            const uint32_t c = static_cast<uint32_t>(kq >> 1);
            mma_mxf4(acc, wdesc0 + wo + 2 * kq, xdesc0 + xo + 2 * kq, hi ? id_hi : id_lo,
                     (t_sfw + 4 * c) | (hi << 31), (t_sfx + 4 * c) | (hi << 31),
                     (s != iss || kq != 0) ? 1u : 0u);
          }
        }
      }
      tc_commit(tmem_full);
    }
  } else {
    // ------------------------------------------------------------ warps 0-3
    // (Xq and its scales are read through L2 only (ld.global.cg): with the flag hand-off
    // they are written by a kernel that is still running.)
    // (1) scales into TMEM: lane l of warp q writes TMEM lane 32q + l, which takes 16-byte
    //     row l of every 512-byte scale chunk (the scales of rows l, l+32, l+64, l+96 of
    //     that chunk's 128-row group), the same for all four lane quarters
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);
    auto put_scales = [&](const uint8_t* group, uint32_t col_off, bool from_l2) {
      uint4 w[kStages][2];  // all loads first: one round trip to memory, not one per stage
#pragma unroll
      for (int s = 0; s < kStages; ++s)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int ch = 2 * (kb + s) + c;
          w[s][c] = make_uint4(0u, 0u, 0u, 0u);
          if (s < nk && ch < p.nbp4) {
            const uint4* src = reinterpret_cast<const uint4*>(group + ch * kChunk) + lane;
            w[s][c] = from_l2 ? __ldcg(src) : __ldg(src);
          }
        }
#pragma unroll
      for (int s = 0; s < kStages; ++s) {
        if (s >= nk) break;
        const uint32_t v[8] = {w[s][0].x, w[s][0].y, w[s][0].z, w[s][0].w,
                               w[s][1].x, w[s][1].y, w[s][1].z, w[s][1].w};
        tmem_st_32x32b_x8(tl + kSfCol0 + kSfStageCols * s + col_off, v);
      }
    };
    const uint8_t* wgroup = p.sfb + tile * p.nbp4 * kChunk;
    if (w_static) put_scales(wgroup, 0, false);
    // Xq, its scales and Y belong to the kernel before
    if (q_flags != nullptr) {
      for (int i = threadIdx.x; i < q_ctas; i += 128) {
        if (ld_acquire_gpu_u64(q_flags + i) == epoch) continue;
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu_u64(q_flags + i) != epoch) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_dev_error, kErrWaitFull);
            break;
          }
          __nanosleep(64);
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four warps: every flag seen
    } else {
      grid_dependency_wait();
    }
    if (!w_static) put_scales(wgroup, 0, false);
    // (2) X codes of all stages: 16-byte chunk j of row r of stage s at
    //     s*nx*128 + r*128 + 16*(j ^ (r % 8)) (the 128-byte swizzle), zeros past M and K;
    //     eight loads per thread in flight at a time, the first eight together with the
    //     X scales' loads
    const int64_t kbytes = p.K / 2;
    const int items = nk * nx * 8;
    uint4 xv[8];
    auto load_x = [&](int i0) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int i = i0 + 128 * t;
        const int j = i & 7;
        const int r = (i >> 3) % nx;
        const int s = (i >> 3) / nx;
        const int64_t col = static_cast<int64_t>(kb + s) * 128 + 16 * j;
        xv[t] = make_uint4(0u, 0u, 0u, 0u);
        if (i < items && r < p.M && col < kbytes)
          xv[t] = __ldcg(reinterpret_cast<const uint4*>(xcodes + static_cast<int64_t>(r) * kbytes + col));
      }
    };
    auto store_x = [&](int i0) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int i = i0 + 128 * t;
        if (i >= items) break;
        const int j = i & 7;
        const int r = (i >> 3) % nx;
        const int s = (i >> 3) / nx;
        st_shared_v4(xbase + s * nx * 128 + r * 128 + ((j ^ (r & 7)) << 4), xv[t].x, xv[t].y,
                     xv[t].z, xv[t].w);
      }
    };
    load_x(threadIdx.x);
    put_scales(p.sfa, 8, true);  // X: the first 128-row group (M <= 64)
    store_x(threadIdx.x);
    for (int i0 = threadIdx.x + 128 * 8; i0 < items; i0 += 128 * 8) {
      load_x(i0);
      store_x(i0);
    }
    fence_proxy_async_smem();  // the stores above are read by the tensor core
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(ready_bar);

    // (3) epilogue: TMEM lane = W row of the tile, columns = tokens
    got = mbar_wait(tmem_full, 0, kErrWaitTmemFull);
    tc_fence_after();
    if (got) {  // (after a stalled wait the accumulator is not read: the output is void anyway)
      tmem_ld_32x32b_x32(tl, r[0]);
      if (nx > 32) tmem_ld_32x32b_x32(tl + 32, r[1]);
      if (nk > 1) {  // the odd stages' accumulator, added second
        uint32_t r2[2][32];
        tmem_ld_32x32b_x32(tl + kAccCols, r2[0]);
        if (nx > 32) tmem_ld_32x32b_x32(tl + kAccCols + 32, r2[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            r[h][c] = __float_as_uint(__uint_as_float(r[h][c]) + __uint_as_float(r2[h][c]));
      }
      tmem_wait_ld();
    }
    if (S > 1) {
      // row rl belongs to rank o: push this rank's partial there, as red[rank][rl - o0][m]
      asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every CTA has started
      const int o = rl * S / kBM;
      if (o != rank) {
        const int o0 = o * kBM / S;
        const uint32_t dst = red + static_cast<uint32_t>((rank * (kBM / S) + (rl - o0)) * kMaxNx * 4);
#pragma unroll
        for (int c = 0; c < kMaxNx / 4; ++c)
          if (4 * c < nx)
            st_async_v4(dst + 16 * (c ^ (rl & 7)), red_bar, static_cast<uint32_t>(o),
                        make_uint4(r[(4 * c) >> 5][(4 * c) & 31], r[(4 * c + 1) >> 5][(4 * c + 1) & 31],
                                   r[(4 * c + 2) >> 5][(4 * c + 2) & 31],
                                   r[(4 * c + 3) >> 5][(4 * c + 3) & 31]));
      }
    }
  }

  if (warp < 4) {
    // (4) this CTA's rows [r0, r0 + nr) of the tile (all 128 when S = 1; the owned share
    //     otherwise) are summed over the S partials in rank order and go to shared memory
    //     as [token][row] in the output type (over the drained W ring), then to Y in
    //     16-byte stores: one per 8 bf16 (4 fp32) outputs, not one per value. The thread
    //     of an owned row first puts its own partial next to the peers' (same swizzled
    //     layout), so that the sum is a rolled loop over shared memory: this code runs
    //     once per launch, and with the benchmark's flushed L2 every new stretch of
    //     straight-line code is fetched from memory.
    const int nr = kBM / S;
    const int r0 = rank * nr;
    const int esz = p.out_f32 ? 4 : 2;
    const uint32_t stage = base;
    const bool own = rl >= r0 && rl < r0 + nr;
    const uint32_t src = red + static_cast<uint32_t>((rl - r0) * kMaxNx * 4);
    if (own) {
      const uint32_t dst = src + static_cast<uint32_t>(rank * nr * kMaxNx * 4);
#pragma unroll
      for (int c = 0; c < kMaxNx / 4; ++c)
        if (4 * c < nx)
          st_shared_v4(dst + 16 * (c ^ (rl & 7)), r[(4 * c) >> 5][(4 * c) & 31],
                       r[(4 * c + 1) >> 5][(4 * c + 1) & 31], r[(4 * c + 2) >> 5][(4 * c + 2) & 31],
                       r[(4 * c + 3) >> 5][(4 * c + 3) & 31]);
    }
    // the peers' partials of the owned rows have landed (every CTA waits for all it is
    // sent, so none exits while a peer still writes into it)
    const bool recv = S == 1 || mbar_wait(red_bar, 0, kErrWaitFull);
    if (got && recv && own) {
      const int nc = static_cast<int>((p.M + 3) / 4);
#pragma unroll 1
      for (int c = 0; c < nc; ++c) {
        const uint32_t cs = static_cast<uint32_t>(4 * (c ^ (rl & 7)) * 4);
        uint4 w = lds_v4_u32(src + cs);
        float a[4] = {__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z),
                      __uint_as_float(w.w)};
#pragma unroll 1
        for (int q = 1; q < S; ++q) {
          w = lds_v4_u32(src + static_cast<uint32_t>(q * nr * kMaxNx * 4) + cs);
          a[0] += __uint_as_float(w.x);
          a[1] += __uint_as_float(w.y);
          a[2] += __uint_as_float(w.z);
          a[3] += __uint_as_float(w.w);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = 4 * c + e;
          if (m >= p.M) break;
          const uint32_t off = static_cast<uint32_t>((m * nr + (rl - r0)) * esz);
          if (p.out_f32)
            sts_b32(stage + off, __float_as_uint(a[e]));
          else
            sts_b16(stage + off, __bfloat16_as_ushort(__float2bfloat16_rn(a[e])));
        }
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four warps: the staged rows
    const int row_bytes = nr * esz;                  // 64..512, a multiple of 16
    const int chunks = row_bytes / 16;
    const int epc = 16 / esz;                        // outputs per chunk
    const int64_t n0 = tile * kBM + r0;
    for (int i = threadIdx.x; i < p.M * chunks; i += 128) {
      const int m = i / chunks;
      const int j = i % chunks;
      const int64_t n = n0 + static_cast<int64_t>(j) * epc;
      const uint4 v = lds_v4_u32(stage + static_cast<uint32_t>(m * row_bytes + j * 16));
      uint8_t* dst = static_cast<uint8_t*>(p.y) + (m * p.N + n) * esz;
      if (p.vec_ok && n + epc <= p.N) {
        stg_v4(dst, v);
      } else {
        for (int e = 0; e < epc; ++e) {
          if (n + e >= p.N) break;
          const int wi = esz == 4 ? e : e >> 1;
          const uint32_t w = wi == 0 ? v.x : wi == 1 ? v.y : wi == 2 ? v.z : v.w;
          if (esz == 4)
            stg_b32(dst + 4 * e, w);
          else
            stg_b16(dst + 2 * e, static_cast<uint16_t>(w >> (16 * (e & 1))));
        }
      }
    }
  }
  // (warps 4-6 complete their part of the cluster barrier too)
  if (S > 1 && warp >= 4) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace bat
