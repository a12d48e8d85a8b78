// Block-scaled MXFP4 GEMM on sm_100a: Y = Xq . Wq^T with UE8M0 scales per 32
// elements along K, the low-bit product Q(XP) . Q(P^-1 W^T) of the BATQuant
// linear layer (BATQuant note, en.papernotes.org, Method > Key Designs 1).
//
// One persistent CTA per SM walks 128 x 256 output tiles. Warp roles (three
// warpgroups; registers are moved to the epilogue with setmaxnreg):
//   warps 0..3  epilogue: tcgen05.ld of the fp32 accumulator, conversion,
//               staged TMA stores of Y (holds a whole bf16 tile row in registers);
//   warps 4..7  scale-factor writers, one per TMEM lane quarter: each stage's
//               scale chunks go shared -> registers -> TMEM (tcgen05.st) into a
//               per-stage TMEM buffer, in the layout the block-scaled MMA reads
//               (each 128-row chunk replicated over the four lane quarters).
//               Writing them from registers keeps the copies off the tensor
//               pipe, where tcgen05.cp would queue behind the MMAs;
//   warp 8      TMA producer: code tiles through 2-D tensor maps (128-byte
//               swizzle) into a ring of kStages shared-memory stages guarded by
//               mbarriers;
//   warp 9      TMEM owner and MMA issuer: tcgen05.mma kind::mxf4.block_scale
//               (M=128, N=256, K=64) accumulating in TMEM;
//               with MXFP8 activations (W4A8, kA8), kind::mxf8f6f4.block_scale
//               (E4M3 x E2M1, K=32), the weights' packed E2M1 codes unpacked by
//               the TMA load into the 16-bytes-per-16-elements layout that MMA reads;
//   warp 10     scale producer: the stage's scale tiles as 1-D bulk copies (the code
//               tiles' producer and this warp split a stage's copy instructions);
//   warp 11     idle (it completes the third warpgroup).
// Every wait is bounded (see mbar_wait) and reports through the error word.
// Launched with programmatic stream serialization, so barrier set-up and the TMEM
// allocation overlap the end of the kernel before it (normally the quantizer).
//
// Split-K for a single row of tiles (M <= 128, few N tiles: the decode shapes).
// With splits = C > 1 the grid is launched in clusters of C CTAs, one cluster per
// tile; CTA r of a cluster takes K stages [r*ks/C, (r+1)*ks/C) and leaves its fp32
// partial tile (valid rows only) in its own shared memory (the drained stage
// buffers). After a cluster barrier each CTA sums, in rank order, one share of the
// tile's 32-column chunks over the C partials it reads through distributed shared
// memory, and writes that share of Y. The sum order is fixed, so the result does
// not depend on timing; a second cluster barrier keeps every partial alive until all
// readers are done.
#pragma once

#include <cooperative_groups.h>

#include "bat_common.cuh"

namespace bat {

namespace gemm {
constexpr int kBM = 128;                     // rows of X per tile (MMA M)
constexpr int kBN = 256;                     // rows of W per tile (MMA N)
constexpr int kStages = 4;
constexpr int kABytes = kBM * 128;           // 16 KB: 128 bytes of codes per row and stage
constexpr int kBBytes = kBN * 128;           // 32 KB
constexpr int kChunk = 512;                  // one 128-row x 4-scale block of the scale layout
constexpr int kThreads = 384;
constexpr uint32_t kRegsEpi = 232;   // after setmaxnreg: 128 x 232 + 256 x 80 <= 384 x 168
constexpr uint32_t kRegsOther = 80;
static_assert(128 * kRegsEpi + 256 * kRegsOther <= kThreads * 168, "register split");
// split-K partial tile in shared memory: fp32 rows of 256 columns, padded to 260 floats
// so that the epilogue's row-per-lane stores spread over the banks
constexpr int kPartStride = kBN + 4;
// bf16 output staging for the TMA store: one box of 128 rows x 64 columns (128 bytes,
// 128-byte swizzle); the epilogue holds its whole bf16 tile in registers and
// streams it through this box one 64-column slice at a time.
constexpr int kEpiBoxBytes = kBM * 128;
constexpr int kEpiBytes = kEpiBoxBytes;  // 16 KB
// Per activation format: K elements per stage (128 bytes of codes per row: 256 packed
// E2M1, or 128 E4M3 with the weights' E2M1 unpacked to a byte each in shared memory),
// the stage's scale chunks, and the stage size (a multiple of 1 KB for the swizzle).
template <bool kA8>
struct Cfg {
  static constexpr int kBK = kA8 ? 128 : 256;
  static constexpr int kChunksPerStage = kBK / 128;                      // 1 or 2
  static constexpr int kSfaBytes = (kBM / 128) * kChunksPerStage * kChunk;
  static constexpr int kSfbBytes = (kBN / 128) * kChunksPerStage * kChunk;
  static constexpr int kStageBytes = (kABytes + kBBytes + kSfaBytes + kSfbBytes + 1023) / 1024 * 1024;
  static constexpr int kSmemBytes = kStages * kStageBytes + kEpiBytes + 1024 /*align*/ + 256 /*barriers*/;
};
// TMEM columns: accumulator [0, 256); stage s's scales at 256 + 24 s: A words
// [0, 8) (up to two 128-K chunks x 4), B words [8, 24) (chunks x two 128-row groups x 4).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;
constexpr uint32_t kSfStageCols = 24;
static_assert(kSfCol0 + kStages * kSfStageCols <= kTmemCols, "TMEM columns");
}  // namespace gemm

struct GemmParams {
  const uint8_t* sfa;  // tiled scales of Xq
  const uint8_t* sfb;  // tiled scales of Wq
  void* y;
  int64_t M, N, K;
  int nbp4;            // ceil(K/32 / 4): scale chunks per 128-row group
  int out_f32;         // 1: fp32 output, 0: bf16
  int vec_ok;          // rows of Y are 16-byte aligned for vector stores
  int tma_store;       // bf16 output written through the staged TMA store
  int splits;          // K splits = cluster size (1: persistent, whole K per tile)
  // CTA-pair kernel, tile-level overlap with the prologue: null (wait for the grid
  // dependency), or the prologue's per-CTA completion flags (q_strips x q_cps CTAs over
  // q_mtiles token tiles and q_nbp2 block pairs), complete when they hold q_epoch
  const unsigned long long* cta_flags;
  int64_t q_mtiles;
  int q_nbp2, q_strips, q_cps;
  unsigned long long q_epoch;
};

__device__ __forceinline__ uint4 lds_v4_u32(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x,
                                             int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
}
// Barrier over the four epilogue warps that also ANDs a flag across them, so that
// all of them take the same branch after a bounded wait (none is left at a barrier).
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void store_chunk(const GemmParams& p, int64_t row, int64_t col0,
                                            const uint32_t (&r)[32]) {
  if (row >= p.M) return;
  const int64_t nvalid = p.N - col0;
  if (nvalid <= 0) return;
  if (p.out_f32) {
    float* dst = static_cast<float*>(p.y) + row * p.N + col0;
    if (p.vec_ok && nvalid >= 32) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        reinterpret_cast<uint4*>(dst)[c] = make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c < nvalid) dst[c] = __uint_as_float(r[c]);
    }
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.y) + row * p.N + col0;
    uint32_t h[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1]));
      h[c] = *reinterpret_cast<uint32_t*>(&v);
    }
    if (p.vec_ok && nvalid >= 32) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        reinterpret_cast<uint4*>(dst)[c] = make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c < nvalid)
          reinterpret_cast<uint16_t*>(dst)[c] = static_cast<uint16_t>(h[c >> 1] >> (16 * (c & 1)));
    }
  }
}

// Sum of the cluster's partial tiles for this CTA's share of the 32-column chunks
// (chunks rank, rank + C, ...), rows of the tile that exist; partials are added in
// rank order 0 .. C-1.
__device__ __forceinline__ void split_reduce(const GemmParams& p, uint8_t* base_ptr,
                                             cooperative_groups::cluster_group& cluster,
                                             int64_t mt, int64_t nt, int rank) {
  using namespace gemm;
  const int C = p.splits;
  const int64_t rows = min(static_cast<int64_t>(kBM), p.M - mt * kBM);
  const int nch = (kBN / 32 - rank + C - 1) / C;  // chunks of this rank
  const int64_t work = rows * nch * 8;             // float4 items
  const float* part = reinterpret_cast<const float*>(base_ptr);
  for (int64_t i = threadIdx.x; i < work; i += blockDim.x) {
    const int64_t row = i / (nch * 8);
    const int j = static_cast<int>(i % (nch * 8));
    const int col = (rank + (j >> 3) * C) * 32 + (j & 7) * 4;  // column within the tile
    const int64_t off = row * kPartStride + col;
    // all C remote loads first (independent, so their latencies overlap), then the sum
    float4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < C) v[q] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(part + off, q));
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < C) {
        acc.x += v[q].x;
        acc.y += v[q].y;
        acc.z += v[q].z;
        acc.w += v[q].w;
      }
    const int64_t m = mt * kBM + row;
    const int64_t n0 = nt * kBN + col;
    const float a[4] = {acc.x, acc.y, acc.z, acc.w};
    if (p.out_f32) {
      float* dst = static_cast<float*>(p.y) + m * p.N + n0;
      if (p.vec_ok && n0 + 4 <= p.N) {
        *reinterpret_cast<float4*>(dst) = acc;
      } else {
        for (int c = 0; c < 4; ++c)
          if (n0 + c < p.N) dst[c] = a[c];
      }
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.y) + m * p.N + n0;
      __nv_bfloat162 lo = __floats2bfloat162_rn(a[0], a[1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(a[2], a[3]);
      if (p.vec_ok && n0 + 4 <= p.N) {
        uint2 w;
        w.x = *reinterpret_cast<uint32_t*>(&lo);
        w.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(dst) = w;
      } else {
        for (int c = 0; c < 4; ++c)
          if (n0 + c < p.N) dst[c] = __float2bfloat16_rn(a[c]);
      }
    }
  }
}

// kA8 = false: Xq MXFP4 (tmap_a over packed codes [M][K/2] bytes).
// kA8 = true:  Xq MXFP8 E4M3 (tmap_a over codes [M][K] bytes) and tmap_b over Wq's packed
//              E2M1 codes with the 16-elements-per-16-bytes shared-memory expansion.
template <bool kA8>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    bat_mxf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  using namespace gemm;
  constexpr int kBK = Cfg<kA8>::kBK;
  constexpr int kChunksPerStage = Cfg<kA8>::kChunksPerStage;
  constexpr int kSfaBytes = Cfg<kA8>::kSfaBytes;
  constexpr int kStageBytes = Cfg<kA8>::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  // stage s: [A 16K][B 32K][SFA 1K][SFB 2K]; then the epilogue staging; then barriers
  const uint32_t stg = base + kStages * kStageBytes;
  const uint32_t bars = stg + kEpiBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
  const uint32_t tmem_full = bars + 8u * (2 * kStages);
  const uint32_t tmem_empty = tmem_full + 8u;
  const uint32_t tmem_slot = tmem_empty + 8u;
  auto sf_bar = [&](int s) { return tmem_slot + 8u + 8u * s; };  // scales of stage s in TMEM
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(base_ptr + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 4);
    for (int s = 0; s < kStages; ++s) mbar_init(sf_bar(s), 4);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    if (p.tma_store) prefetch_tmap(&tmap_y);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  // Everything above is local setup; the operands (and Y) belong to the kernels before.
  grid_dependency_wait();

  const int64_t m_tiles = (p.M + kBM - 1) / kBM;
  const int64_t n_tiles = (p.N + kBN - 1) / kBN;
  const int64_t tiles = m_tiles * n_tiles;
  const int k_stages = static_cast<int>((p.K + kBK - 1) / kBK);
  // the tiles this CTA visits and its K stages [kb, ke): with split-K one tile per
  // cluster and a slice of K per cluster rank; otherwise a persistent walk over tiles
  const bool split = p.splits > 1;
  const int rank = split ? static_cast<int>(blockIdx.x % p.splits) : 0;
  const int64_t tile0 = split ? blockIdx.x / p.splits : blockIdx.x;
  const int64_t tstride = split ? tiles : gridDim.x;
  const int kb = split ? rank * k_stages / p.splits : 0;
  const int ke = split ? (rank + 1) * k_stages / p.splits : k_stages;
  const int64_t sf_groups_b = (p.N + 127) / 128;
  bool ok = true;

  if (warp >= 8) {
    setmaxnreg_dec<kRegsOther>();  // warpgroup 2: producer, MMA issuer, two idle warps
  }
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t inflight = 0;  // bit s: stage s was loaded; bit 16+s: parity of that load
      for (int64_t tile = tile0; tile < tiles && ok; tile += tstride) {
        const int64_t mt = tile % m_tiles;
        const int64_t nt = tile / m_tiles;
        const int ngb = (nt * 2 + 1 < sf_groups_b) ? 2 : 1;  // 128-row scale groups of this W tile
        for (int ks = kb; ks < ke; ++ks) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          const int c0 = ks * kChunksPerStage;
          const int nch = min(kChunksPerStage, p.nbp4 - c0);
          // the unpacking load of W (kA8) moves 64 bytes per row: its 8-byte gaps in shared
          // memory are not written and count no transaction bytes
          constexpr uint32_t kBTx = kA8 ? kBBytes / 2 : kBBytes;
          const uint32_t bytes = kABytes + kBTx + static_cast<uint32_t>(nch) * kChunk * (1 + ngb);
          const uint32_t sa = base + stage * kStageBytes;
          // the expected bytes include the scale copies warp 10 issues (their completions may
          // come first: the phase still waits for this arrival)
          mbar_expect_tx(full_bar(stage), bytes);
          // x of both maps is 128 per stage: bytes of packed E2M1, E4M3 elements, or
          // (unpacking load) E2M1 elements
          tma_load_2d(sa, &tmap_a, full_bar(stage), ks * 128, static_cast<int32_t>(mt * kBM));
          tma_load_2d(sa + kABytes, &tmap_b, full_bar(stage), ks * 128,
                      static_cast<int32_t>(nt * kBN));
          inflight = (inflight & ~(0x10001u << stage)) | (1u << stage) | (phase << (16 + stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // No copy may still be writing shared memory when the CTA exits: wait (bounded) for
      // the last load of every stage. Its phase completes when all five copies of the stage
      // (this warp's code tiles and warp 10's scale chunks, counted together) have landed,
      // so this also covers the scale producer's copies of the stage.
      for (int s = 0; s < kStages; ++s)
        if ((inflight >> s) & 1u) mbar_wait(full_bar(s), (inflight >> (16 + s)) & 1u, kErrWaitFull);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ scale producer
    // Each copy instruction costs the issuing thread some 60-120 cycles; the scale copies
    // go out from this warp so that one stage's copies are issued in about half the time.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t inflight = 0;  // as in the code producer
      for (int64_t tile = tile0; tile < tiles && ok; tile += tstride) {
        const int64_t mt = tile % m_tiles;
        const int64_t nt = tile / m_tiles;
        const int ngb = (nt * 2 + 1 < sf_groups_b) ? 2 : 1;
        for (int ks = kb; ks < ke; ++ks) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          const int c0 = ks * kChunksPerStage;
          const int nch = min(kChunksPerStage, p.nbp4 - c0);
          const uint32_t sa = base + stage * kStageBytes;
          bulk_load(sa + kABytes + kBBytes, p.sfa + (mt * p.nbp4 + c0) * kChunk, nch * kChunk,
                    full_bar(stage));
          for (int g = 0; g < ngb; ++g)
            bulk_load(sa + kABytes + kBBytes + kSfaBytes + g * (kChunksPerStage * kChunk),
                      p.sfb + ((nt * 2 + g) * p.nbp4 + c0) * kChunk, nch * kChunk, full_bar(stage));
          inflight = (inflight & ~(0x10001u << stage)) | (1u << stage) | (phase << (16 + stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // the same bounded drain for this warp's copies
      for (int s = 0; s < kStages; ++s)
        if ((inflight >> s) & 1u) mbar_wait(full_bar(s), (inflight >> (16 + s)) & 1u, kErrWaitFull);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors of stage 0; other stages and K sub-blocks only move the start
      // address field (bits 0-13, in 16-byte units), so a plain add suffices.
      const uint64_t adesc0 = smem_desc(base, 16, 1024, 2);
      const uint64_t bdesc0 = smem_desc(base + kABytes, 16, 1024, 2);
      constexpr uint32_t kStageU = kStageBytes >> 4;
      const uint32_t id_lo = idesc_mxf4(kBM, kBN, 0, 0);  // scale bytes 0-1 of each word
      const uint32_t id_hi = idesc_mxf4(kBM, kBN, 2, 2);  // scale bytes 2-3
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      for (int64_t tile = tile0; tile < tiles && ok; tile += tstride) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1u, kErrWaitTmemEmpty)) { ok = false; break; }
        tc_fence_after();
        for (int ks = kb; ks < ke; ++ks) {
          if (!mbar_wait(full_bar(stage), phase, kErrWaitFull) ||
              !mbar_wait(sf_bar(stage), phase, kErrWaitFull)) { ok = false; break; }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(stage) * kStageU;
          const uint32_t t_sfa = tmem_base + kSfCol0 + kSfStageCols * stage;
          const uint32_t t_sfb = t_sfa + 8;
          const int64_t krem = p.K - static_cast<int64_t>(ks) * kBK;
          const uint32_t acc0 = (ks != kb) ? 1u : 0u;
          if constexpr (kA8) {
            // four K=32 MMAs, 32 bytes of each operand apiece; scale byte c of each word
            // (K % 128 == 0, so every stage is full)
#pragma unroll
            for (uint32_t c = 0; c < 4; ++c)
              mma_mxf8f6f4(tmem_base, adesc0 + so + 2 * c, bdesc0 + so + 2 * c,
                           idesc_mxf8f6f4_e4m3_e2m1(kBM, kBN, c, c), t_sfa | (c << 30),
                           t_sfb | (c << 30), (acc0 | c) != 0 ? 1u : 0u);
          } else if (krem >= kBK) {
            // four K=64 MMAs; 32 bytes of codes each; scale byte pair 0-1 then 2-3 of each chunk
            mma_mxf4(tmem_base, adesc0 + so, bdesc0 + so, id_lo, t_sfa, t_sfb, acc0);
            mma_mxf4(tmem_base, adesc0 + so + 2, bdesc0 + so + 2, id_hi, t_sfa | (2u << 30),
                     t_sfb | (2u << 30), 1u);
            mma_mxf4(tmem_base, adesc0 + so + 4, bdesc0 + so + 4, id_lo, t_sfa + 4, t_sfb + 8, 1u);
            mma_mxf4(tmem_base, adesc0 + so + 6, bdesc0 + so + 6, id_hi, (t_sfa + 4) | (2u << 30),
                     (t_sfb + 8) | (2u << 30), 1u);
          } else {
            const int nkb = static_cast<int>((krem + 63) / 64);
            for (int kb = 0; kb < nkb; ++kb) {
              const uint32_t hi = static_cast<uint32_t>(kb & 1);
              const uint32_t c = static_cast<uint32_t>(kb >> 1);
              mma_mxf4(tmem_base, adesc0 + so + 2 * kb, bdesc0 + so + 2 * kb, hi ? id_hi : id_lo,
                       (t_sfa + 4 * c) | (hi << 31), (t_sfb + 8 * c) | (hi << 31),
                       (acc0 | static_cast<uint32_t>(kb)) != 0 ? 1u : 0u);
            }
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        tc_commit(tmem_full);
        acc_phase ^= 1u;
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ scale-factor writers
    setmaxnreg_dec<kRegsOther>();
    // Warp w writes TMEM lane quarter q = w % 4. Lane l of it holds TMEM lane 32q + l,
    // which takes 16-byte row l of every 512-byte chunk (the scales of rows l, l+32,
    // l+64, l+96 of that chunk's 128-row group) at the chunk's four words.
    const int q = warp & 3;
    const uint32_t tlane = static_cast<uint32_t>(32 * q) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int64_t tile = tile0; tile < tiles && ok; tile += tstride) {
      for (int ks = kb; ks < ke; ++ks) {
        if (!mbar_wait(full_bar(stage), phase, kErrWaitFull)) { ok = false; break; }
        const uint32_t ssf = base + stage * kStageBytes + kABytes + kBBytes + lane * 16;
        uint32_t fa[8] = {}, fb[16] = {};
#pragma unroll
        for (int c = 0; c < kChunksPerStage; ++c) {
          const uint4 v = lds_v4_u32(ssf + c * kChunk);
          fa[4 * c] = v.x; fa[4 * c + 1] = v.y; fa[4 * c + 2] = v.z; fa[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int c = 0; c < kChunksPerStage; ++c)
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const uint4 v = lds_v4_u32(ssf + kSfaBytes + g * (kChunksPerStage * kChunk) + c * kChunk);
            const int w = 8 * c + 4 * g;
            fb[w] = v.x; fb[w + 1] = v.y; fb[w + 2] = v.z; fb[w + 3] = v.w;
          }
        const uint32_t tcol = tmem_base + tlane + kSfCol0 + kSfStageCols * stage;
        tmem_st_32x32b_x8(tcol, fa);
        if constexpr (kA8) {
          uint32_t fb8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) fb8[i] = fb[i];
          tmem_st_32x32b_x8(tcol + 8, fb8);
        } else {
          tmem_st_32x32b_x16(tcol + 8, fb);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_bar(stage));
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int rl = 32 * q + lane;  // row within the tile
    const bool leader = (warp == 0 && lane == 0);
    uint32_t acc_phase = 0;
    for (int64_t tile = tile0; tile < tiles && ok; tile += tstride) {
      const int64_t mt = tile % m_tiles;
      const int64_t nt = tile / m_tiles;
      bool got = mbar_wait(tmem_full, acc_phase, kErrWaitTmemFull);
      if (p.tma_store) got = epi_bar_and(got);
      if (!got) { ok = false; break; }
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      if (split) {
        // partial tile -> this CTA's shared memory (rows of the tile that exist); every
        // stage has been consumed by the MMAs that tmem_full waited for
        const bool row_ok = mt * kBM + rl < p.M;
        const uint32_t prow = base + static_cast<uint32_t>(rl * kPartStride * 4);
#pragma unroll 1
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + cc * 32, r);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(prow + (cc * 32 + 4 * j) * 4, r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_empty);
      } else if (p.tma_store) {
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
        if (lane == 0) mbar_arrive(tmem_empty);  // accumulator free: next tile's MMAs may start
        // 2) stream 64-column slices through the staging box; 16-byte chunk j of row rl
        //    sits at chunk (j ^ (rl % 8)) (the 128-byte swizzle of the store's tensor map)
        const uint32_t rowb = stg + rl * 128;
#pragma unroll
        for (int b = 0; b < kBN / 64; ++b) {
          if (leader) bulk_wait_read0();  // the previous slice has left the box
          epi_bar_sync();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(rowb + ((j ^ (rl & 7)) << 4), h[b * 32 + 4 * j], h[b * 32 + 4 * j + 1],
                         h[b * 32 + 4 * j + 2], h[b * 32 + 4 * j + 3]);
          fence_async_smem();
          epi_bar_sync();
          const int64_t col = nt * kBN + 64 * b;
          if (leader && col < p.N) {
            tma_store_2d(&tmap_y, stg, static_cast<int32_t>(col), static_cast<int32_t>(mt * kBM));
            bulk_commit();
          }
        }
      } else {
        const int64_t row = mt * kBM + rl;
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + cc * 32, r);
          tmem_wait_ld();
          store_chunk(p, row, nt * kBN + cc * 32, r);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_empty);
      }
      acc_phase ^= 1u;
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (split) {
    // every CTA of the cluster reaches both barriers, error or not
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // all partials written
    split_reduce(p, base_ptr, cluster, tile0 % m_tiles, tile0 / m_tiles, rank);
    cluster.sync();  // all partials read
  }
  if (warp == 9) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace bat
