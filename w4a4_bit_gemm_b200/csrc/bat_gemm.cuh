// Block-scaled MXFP4 GEMM on sm_100a: Y = Xq . Wq^T with UE8M0 scales per 32
// elements along K, the low-bit product Q(XP) . Q(P^-1 W^T) of the BATQuant
// linear layer (BATQuant note, en.papernotes.org, Method > Key Designs 1).
//
// One persistent CTA per SM walks 128 x 256 output tiles. Warp roles:
//   warp 0      TMA producer: code tiles through 2-D tensor maps (128-byte
//               swizzle), scale tiles through 1-D bulk copies, into a ring of
//               kStages shared-memory stages guarded by mbarriers;
//   warp 1      TMEM owner and MMA issuer: copies each stage's scale factors
//               shared -> TMEM (tcgen05.cp, replicated over the four lane
//               quarters) and issues tcgen05.mma kind::mxf4.block_scale
//               (M=128, N=256, K=64) accumulating in TMEM;
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, conversion,
//               stores of Y.
// Every wait is bounded (see mbar_wait) and reports through the error word.
#pragma once

#include "bat_common.cuh"

namespace bat {

namespace gemm {
constexpr int kBM = 128;                     // rows of X per tile (MMA M)
constexpr int kBN = 256;                     // rows of W per tile (MMA N)
constexpr int kBK = 256;                     // K elements per stage (128 bytes of codes per row)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK / 2;       // 16 KB
constexpr int kBBytes = kBN * kBK / 2;       // 32 KB
constexpr int kChunk = 512;                  // one 128-row x 4-scale block of the scale layout
constexpr int kChunksPerStage = kBK / 128;   // 2
constexpr int kSfaBytes = (kBM / 128) * kChunksPerStage * kChunk;  // 1 KB
constexpr int kSfbBytes = (kBN / 128) * kChunksPerStage * kChunk;  // 2 KB
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kThreads = 192;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
// TMEM columns: accumulator [0, 256), A scales [256, 264), B scales [264, 280).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = 256;
constexpr uint32_t kSfbCol = 264;
}  // namespace gemm

struct GemmParams {
  const uint8_t* sfa;  // tiled scales of Xq
  const uint8_t* sfb;  // tiled scales of Wq
  void* y;
  int64_t M, N, K;
  int nbp4;            // ceil(K/32 / 4): scale chunks per 128-row group
  int out_f32;         // 1: fp32 output, 0: bf16
  int vec_ok;          // rows of Y are 16-byte aligned for vector stores
};

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

__global__ void __launch_bounds__(gemm::kThreads, 1)
    bat_mxf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b, const GemmParams p) {
  using namespace gemm;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  // stage s: [A 16K][B 32K][SFA 1K][SFB 2K]
  const uint32_t bars = base + kStages * kStageBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
  const uint32_t tmem_full = bars + 8u * (2 * kStages);
  const uint32_t tmem_empty = tmem_full + 8u;
  const uint32_t tmem_slot = tmem_empty + 8u;
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
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;

  const int64_t m_tiles = (p.M + kBM - 1) / kBM;
  const int64_t n_tiles = (p.N + kBN - 1) / kBN;
  const int64_t tiles = m_tiles * n_tiles;
  const int k_stages = static_cast<int>((p.K + kBK - 1) / kBK);
  const int64_t sf_groups_b = (p.N + 127) / 128;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int64_t mt = tile % m_tiles;
        const int64_t nt = tile / m_tiles;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          const int c0 = ks * kChunksPerStage;
          const int nch = min(kChunksPerStage, p.nbp4 - c0);
          int ngb = 0;
          for (int g = 0; g < kBN / 128; ++g) ngb += (nt * 2 + g < sf_groups_b) ? 1 : 0;
          const uint32_t bytes = kABytes + kBBytes + static_cast<uint32_t>(nch) * kChunk * (1 + ngb);
          const uint32_t sa = base + stage * kStageBytes;
          mbar_expect_tx(full_bar(stage), bytes);
          tma_load_2d(sa, &tmap_a, full_bar(stage), ks * (kBK / 2), static_cast<int32_t>(mt * kBM));
          tma_load_2d(sa + kABytes, &tmap_b, full_bar(stage), ks * (kBK / 2),
                      static_cast<int32_t>(nt * kBN));
          bulk_load(sa + kABytes + kBBytes, p.sfa + (mt * p.nbp4 + c0) * kChunk, nch * kChunk,
                    full_bar(stage));
          for (int g = 0; g < kBN / 128; ++g) {
            const int64_t grp = nt * 2 + g;
            if (grp < sf_groups_b)
              bulk_load(sa + kABytes + kBBytes + kSfaBytes + g * (kChunksPerStage * kChunk),
                        p.sfb + (grp * p.nbp4 + c0) * kChunk, nch * kChunk, full_bar(stage));
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int64_t nt = tile / m_tiles;
        if (!mbar_wait(tmem_empty, acc_phase ^ 1u, kErrWaitTmemEmpty)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(full_bar(stage), phase, kErrWaitFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t sb = sa + kABytes;
          const uint32_t ssfa = sb + kBBytes;
          const uint32_t ssfb = ssfa + kSfaBytes;
          const int c0 = ks * kChunksPerStage;
          const int nch = min(kChunksPerStage, p.nbp4 - c0);
          for (int c = 0; c < nch; ++c) {
            tmem_cp_32x128b_x4(tmem_base + kSfaCol + 4 * c, smem_desc(ssfa + c * kChunk, 0, 128, 0));
            for (int g = 0; g < kBN / 128; ++g)
              if (nt * 2 + g < sf_groups_b)
                tmem_cp_32x128b_x4(tmem_base + kSfbCol + 8 * c + 4 * g,
                                   smem_desc(ssfb + g * (kChunksPerStage * kChunk) + c * kChunk, 0, 128, 0));
          }
          const int64_t krem = p.K - static_cast<int64_t>(ks) * kBK;
          const int nkb = krem >= 256 ? 4 : static_cast<int>((krem + 63) / 64);
          for (int kb = 0; kb < nkb; ++kb) {
            const uint32_t sf_id = (kb & 1) * 2;
            const uint32_t c = kb >> 1;
            const uint64_t adesc = smem_desc(sa + kb * 32, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(sb + kb * 32, 16, 1024, 2);
            const uint32_t idesc = idesc_mxf4(kBM, kBN, sf_id, sf_id);
            const uint32_t sfa_addr = (tmem_base + kSfaCol + 4 * c) | (sf_id << 30);
            const uint32_t sfb_addr = (tmem_base + kSfbCol + 8 * c) | (sf_id << 30);
            mma_mxf4(tmem_base, adesc, bdesc, idesc, sfa_addr, sfb_addr, (ks | kb) != 0);
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        tc_commit(tmem_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      const int64_t mt = tile % m_tiles;
      const int64_t nt = tile / m_tiles;
      if (!mbar_wait(tmem_full, acc_phase, kErrWaitTmemFull)) { ok = false; break; }
      tc_fence_after();
      const int64_t row = mt * kBM + 32 * q + lane;
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + cc * 32, r);
        tmem_wait_ld();
        store_chunk(p, row, nt * kBN + cc * 32, r);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
      acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace bat
