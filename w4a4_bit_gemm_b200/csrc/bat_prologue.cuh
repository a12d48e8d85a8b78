// Fused prologue: GPK block transform + block-wise clipping + MXFP4 quantize/pack.
//
// BATQuant note (en.papernotes.org), Method > Key Designs 2 and 3: each
// 32-channel block x (a row-major 4x8 matrix X_r) becomes
// y = vec_row(B_b^T X_r A) — two small matrix products instead of the explicit
// 32x32 block B_b (x) A — then is clipped to [r_lo*min(y), r_hi*max(y)] and
// quantized to E2M1 codes with one UE8M0 scale 2^e, e = floor(log2 amax) - 2.
//
// Work mapping. X is cut into segments of 32 consecutive blocks (1024 columns,
// 2 KB of bf16 per row). A CTA owns one segment and a range of rows, so each
// lane owns one fixed block b for the whole kernel: the shared factor A
// (fp32 column pairs) and the lane's private factor B_b (broadcast pairs) are
// loaded into registers once. One producer warp streams the CTA's rows into a
// ring of shared-memory stages with bulk copies (8 rows x 2 KB per stage);
// eight consumer warps each take one row of a stage, lane = block. A lane reads
// its 64 bytes as four 16-byte chunks (rows of X_r) in a rotated order so that
// the eight lanes of each shared-memory phase hit distinct banks; the rotation
// is undone by permuting the rows of B_b once. The transform runs on packed
// fp32x2 FMAs; min/max, clip bounds, scale and codes stay in registers; each
// lane stores 16 bytes of codes (a warp writes 512 contiguous bytes) and its
// scale byte into the tiled order the GEMM reads.
#pragma once

#include "bat_common.cuh"

namespace bat {

namespace pro {
constexpr int kRowsPerStage = 8;                 // = consumer warps
constexpr int kStages = 4;
constexpr int kSegBytes = 32 * kG * 2;           // 2 KB: 32 blocks of 32 bf16
constexpr int kStageBytes = kRowsPerStage * kSegBytes;
constexpr int kThreads = 32 * (kRowsPerStage + 1);
constexpr int kSmemBytes = kStages * kStageBytes + 128;
}  // namespace pro

struct PrologueParams {
  const uint16_t* x;     // bf16 [rows][K]
  const float* a;        // fp32 [8][8]
  const float* b;        // fp32 [nb][4][4]
  const float* g_lo;     // clip logits: [nb] (shared by rows) or [rows][nb]; may be null
  const float* g_hi;
  uint8_t* codes;        // [rows][K/2]
  uint8_t* scales;       // tiled, rows padded to 128, blocks padded to 4
  float* y_out;          // optional fp32 [rows][K] trace of the transformed values
  int64_t rows;
  int64_t K;
  int nb;                // K / 32
  int nseg;              // ceil(nb / 32)
  int nbp4;              // ceil(nb / 4)
  int64_t rows_per_cta;  // rows of one segment handled by one CTA
};

// fp32(sigma(g)) evaluated in fp64; +inf gives exactly 1.
__device__ __forceinline__ float clip_ratio(float g) {
  if (isinf(g) && g > 0.0f) return 1.0f;
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(g))));
}

__device__ __forceinline__ int64_t scale_offset(int64_t m, int64_t b, int nbp4) {
  return ((m >> 7) * nbp4 + (b >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (b & 3);
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

// kPerRowClip: clip logits indexed [row][block] (weight side) instead of [block].
template <bool kTrace, bool kPerRowClip>
__global__ void __launch_bounds__(pro::kThreads, 1) bat_prologue_kernel(const PrologueParams p) {
  using namespace pro;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kStages * kStageBytes;  // full[s], empty[s]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;

  const int seg = static_cast<int>(blockIdx.x % p.nseg);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x / p.nseg) * p.rows_per_cta;
  const int64_t row1 = min(p.rows, row0 + p.rows_per_cta);
  const int nblk = min(32, p.nb - seg * 32);           // blocks in this segment
  const uint32_t seg_bytes = static_cast<uint32_t>(nblk) * kG * 2;
  const int nst = row1 > row0 ? static_cast<int>((row1 - row0 + kRowsPerStage - 1) / kRowsPerStage) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + 8 * s, 1);
      mbar_init(bars + 8 * (kStages + s), kRowsPerStage);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == kRowsPerStage) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int st = 0; st < nst; ++st) {
        const int slot = st % kStages;
        const uint32_t par = static_cast<uint32_t>((st / kStages) & 1);
        if (!mbar_wait(bars + 8 * (kStages + slot), par ^ 1u, kErrWaitEmpty)) break;
        const int64_t r0 = row0 + static_cast<int64_t>(st) * kRowsPerStage;
        const int nrows = row1 - r0 < kRowsPerStage ? static_cast<int>(row1 - r0) : kRowsPerStage;
        mbar_expect_tx(bars + 8 * slot, seg_bytes * nrows);
        for (int r = 0; r < nrows; ++r)
          bulk_load(sbase + slot * kStageBytes + r * kSegBytes,
                    p.x + (r0 + r) * p.K + static_cast<int64_t>(seg) * 1024, seg_bytes, bars + 8 * slot);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int b = seg * 32 + lane;
    const bool active = lane < nblk;
    const int rot = (lane >> 1) & 3;  // chunk rotation: conflict-free 16-byte shared loads
    // Shared factor A as packed column pairs: a2[p][qq] = {A[p][2qq], A[p][2qq+1]}.
    uint64_t a2[8][4];
#pragma unroll
    for (int pp = 0; pp < 8; ++pp)
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const float2 v = reinterpret_cast<const float2*>(p.a)[pp * 4 + qq];
        a2[pp][qq] = pack2(v.x, v.y);
      }
    // Private factor with rows rotated like the chunks: b2[i'][j] = {B[(i'+rot)%4][j], same}.
    uint64_t b2[4][4];
    float r_lo = 1.0f, r_hi = 1.0f;
    {
      const float4* bp = reinterpret_cast<const float4*>(p.b + static_cast<int64_t>(active ? b : 0) * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(bp + ((i + rot) & 3));
        b2[i][0] = pack2(v.x, v.x);
        b2[i][1] = pack2(v.y, v.y);
        b2[i][2] = pack2(v.z, v.z);
        b2[i][3] = pack2(v.w, v.w);
      }
      if (!kPerRowClip && active) {
        r_lo = p.g_lo ? clip_ratio(p.g_lo[b]) : 1.0f;
        r_hi = p.g_hi ? clip_ratio(p.g_hi[b]) : 1.0f;
      }
    }

    for (int st = 0; st < nst; ++st) {
      const int slot = st % kStages;
      const uint32_t par = static_cast<uint32_t>((st / kStages) & 1);
      if (!mbar_wait(bars + 8 * slot, par, kErrWaitFull)) break;
      const int64_t m = row0 + static_cast<int64_t>(st) * kRowsPerStage + warp;
      if (m < row1 && active) {
        if (kPerRowClip) {
          const int64_t ri = m * p.nb + b;
          r_lo = p.g_lo ? clip_ratio(p.g_lo[ri]) : 1.0f;
          r_hi = p.g_hi ? clip_ratio(p.g_hi[ri]) : 1.0f;
        }
        const uint32_t src = sbase + slot * kStageBytes + warp * kSegBytes + lane * 64;
        // ---- T' = X_r' A, where X_r' row i' is chunk (i' + rot) % 4 of the block
        uint64_t t2[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = lds_v4(src + (((i + rot) & 3) << 4));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) t2[i][qq] = 0ull;
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) {
            const uint32_t word = w4[pp >> 1];
            const float xv = (pp & 1) ? bf16hi(word) : bf16lo(word);
            const uint64_t xx = pack2(xv, xv);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) t2[i][qq] = ffma2(xx, a2[pp][qq], t2[i][qq]);
          }
        }
        // ---- Y = B^T T = sum_i' B'[i'][j] T'[i']
        float y[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            uint64_t acc = fmul2(b2[0][j], t2[0][qq]);
            acc = ffma2(b2[1][j], t2[1][qq], acc);
            acc = ffma2(b2[2][j], t2[2][qq], acc);
            acc = ffma2(b2[3][j], t2[3][qq], acc);
            unpack2(acc, y[8 * j + 2 * qq], y[8 * j + 2 * qq + 1]);
          }
        }
        const int64_t eoff = m * p.K + static_cast<int64_t>(b) * kG;  // element offset of the block
        if (kTrace) {
          float4* dst = reinterpret_cast<float4*>(p.y_out + eoff);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
        }
        // ---- block clip: [r_lo * min, r_hi * max]
        // pairwise trees (depth 5) instead of 31-long dependency chains
        float tmn[16], tmx[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          tmn[k] = fminf(y[2 * k], y[2 * k + 1]);
          tmx[k] = fmaxf(y[2 * k], y[2 * k + 1]);
        }
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) {
            tmn[k] = fminf(tmn[k], tmn[k + w]);
            tmx[k] = fmaxf(tmx[k], tmx[k + w]);
          }
        const float mn = tmn[0], mx = tmx[0];
        const float lo = __fmul_rn(r_lo, mn);
        const float hi = __fmul_rn(r_hi, mx);
        // The clamp is monotone, so the clipped block's extremes are the clipped min/max.
        const float amax = fmaxf(fabsf(fminf(fmaxf(mn, lo), hi)), fabsf(fminf(fmaxf(mx, lo), hi)));
        // ---- UE8M0 scale: e = floor(log2 amax) - 2, clamped to >= -127 (amax = 0 -> -127)
        const int efield = static_cast<int>(__float_as_uint(amax) >> 23);
        const int sbyte = efield > 2 ? efield - 2 : 0;  // e + 127
        const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);  // 2^-e
        const uint64_t s2 = pack2(inv_scale, inv_scale);
        // ---- codes: v = c * 2^-e (+0 turns an exact -0 into +0), E2M1 round-to-nearest-even
        uint32_t byte[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float c0 = fminf(fmaxf(y[2 * h], lo), hi);
          const float c1 = fminf(fmaxf(y[2 * h + 1], lo), hi);
          float v0, v1;
          unpack2(ffma2(pack2(c0, c1), s2, 0ull), v0, v1);
          byte[h] = e2m1x2(v0, v1);
        }
        uint32_t packed[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          packed[c] = (byte[4 * c] | (byte[4 * c + 1] << 8)) | ((byte[4 * c + 2] << 16) | (byte[4 * c + 3] << 24));
        *reinterpret_cast<uint4*>(p.codes + eoff / 2) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        p.scales[scale_offset(m, b, p.nbp4)] = static_cast<uint8_t>(sbyte);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (kStages + slot));
    }
  }

  // ---- zero the padding bytes of the tiled scale buffer
  const int64_t rows_pad = (p.rows + 127) & ~static_cast<int64_t>(127);
  const int64_t bcols = static_cast<int64_t>(p.nbp4) * 4;
  const int64_t pad_cols = bcols - p.nb;                // blocks past nb, rows < M
  const int64_t n_right = p.rows * pad_cols;
  const int64_t n_below = (rows_pad - p.rows) * bcols;  // rows past M, all blocks
  const int64_t tstride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       t < n_right + n_below; t += tstride) {
    int64_t m, bb;
    if (t < n_right) {
      m = t / pad_cols;
      bb = p.nb + (t - m * pad_cols);
    } else {
      const int64_t r = t - n_right;
      m = p.rows + r / bcols;
      bb = r - (m - p.rows) * bcols;
    }
    p.scales[scale_offset(m, bb, p.nbp4)] = 0;
  }
}

__global__ void bat_clip_ratio_kernel(const float* g, int64_t n, float* r) {
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    r[t] = g ? clip_ratio(g[t]) : 1.0f;
}

}  // namespace bat
