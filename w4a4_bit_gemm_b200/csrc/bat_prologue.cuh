// Fused prologue: GPK block transform + block-wise clipping + MXFP4 quantize/pack.
//
// BATQuant note (en.papernotes.org), Method > Key Designs 2 and 3: each
// 32-channel block x (a row-major 4x8 matrix X_r) becomes
// y = vec_row(B_b^T X_r A) — two small matrix products instead of the explicit
// 32x32 block B_b (x) A — then is clipped to [r_lo*min(y), r_hi*max(y)] and
// quantized to E2M1 codes with one UE8M0 scale 2^e, e = floor(log2 amax) - 2.
//
// Work mapping. X is cut into segments of 32 consecutive blocks (1024 columns,
// 2 KB of bf16 per row). A CTA owns one segment and a range of rows. One
// producer warp streams the CTA's rows into a ring of shared-memory stages
// with bulk copies (16 rows x 2 KB per stage); each of 16 consumer warps takes
// one row of a stage.
//  1. T = X_r A for all 128 rows of 8 of the segment (the shared factor is the
//     same for every block) runs on the tensor cores: ldmatrix feeds the 16-byte
//     rows straight from the stage to mma.sync (bf16 inputs, fp32 accumulate).
//     x is exact in bf16; A is split into three bf16 terms A_hi + A_mid + A_lo
//     (residual ~2^-24 |A|), so T matches an fp32 product to within fp32 rounding.
//  2. The 16x8 accumulator fragments go to a per-warp shared buffer, swizzled
//     so that lane b then reads block b's 4x8 T with conflict-free 16-byte loads.
//  3. Per lane (= block): Y = B_b^T T on packed fp32x2 FMAs (B_b as broadcast
//     pairs in registers), block min/max by 3-input min/max trees, clip bounds,
//     scale and E2M1 codes in registers; 16 bytes of codes per lane (a warp
//     writes 512 contiguous bytes) and one scale byte in the GEMM's tiled order.
#pragma once

#include "bat_common.cuh"

namespace bat {

namespace pro {
constexpr int kRowsPerStage = 16;                // = consumer warps
constexpr int kStages = 5;
constexpr int kSegBytes = 32 * kG * 2;           // 2 KB: 32 blocks of 32 bf16
constexpr int kStageBytes = kRowsPerStage * kSegBytes;
constexpr int kTBytes = 32 * 32 * 4;             // per-warp fp32 T of one segment: 4 KB
constexpr int kThreads = 32 * (kRowsPerStage + 1);
constexpr int kSmemBytes = kStages * kStageBytes + kRowsPerStage * kTBytes + 256;
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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A(16x16, rows g / g+8) . B(16x8) + C, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
__device__ __forceinline__ void sts_v2(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// bf16 (round-to-nearest-even) of an fp32 value, as raw bits.
__device__ __forceinline__ uint32_t bf16_bits(float v) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
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
    const int g = lane >> 2;  // mma fragment coordinates
    const int t4 = lane & 3;
    // Shared factor for the tensor-core stage: B-operand fragments of A split into
    // three bf16 terms. Fragment (k = 2*t4 + {0,1}, n = g): A[2*t4 + {0,1}][g].
    uint32_t fa_hm0, fa_hm1, fa_lo;
    {
      const float v0 = p.a[(2 * t4) * 8 + g], v1 = p.a[(2 * t4 + 1) * 8 + g];
      const uint32_t h0 = bf16_bits(v0), h1 = bf16_bits(v1);
      const float r0 = v0 - __uint_as_float(h0 << 16), r1 = v1 - __uint_as_float(h1 << 16);
      const uint32_t m0 = bf16_bits(r0), m1 = bf16_bits(r1);
      const float s0 = r0 - __uint_as_float(m0 << 16), s1 = r1 - __uint_as_float(m1 << 16);
      fa_hm0 = h0 | (h1 << 16);                    // k 0-7 of the k16 MMA: A_hi
      fa_hm1 = m0 | (m1 << 16);                    // k 8-15: A_mid
      fa_lo = bf16_bits(s0) | (bf16_bits(s1) << 16);  // the k8 MMA: A_lo
    }
    // Private factor as broadcast pairs: b2[i][j] = {B[i][j], B[i][j]}.
    uint64_t b2[4][4];
    float r_lo = 1.0f, r_hi = 1.0f;
    {
      const float4* bp = reinterpret_cast<const float4*>(p.b + static_cast<int64_t>(active ? b : 0) * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(bp + i);
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
    const uint32_t tbuf = sbase + kStages * kStageBytes + warp * kTBytes;

    for (int st = 0; st < nst; ++st) {
      const int slot = st % kStages;
      const uint32_t par = static_cast<uint32_t>((st / kStages) & 1);
      if (!mbar_wait(bars + 8 * slot, par, kErrWaitFull)) break;
      const int64_t m = row0 + static_cast<int64_t>(st) * kRowsPerStage + warp;
      const bool row_ok = m < row1;
      if (row_ok) {
        // ---- 1+2: T = X_r A on the tensor cores, 16 rows of 8 (4 blocks) per MMA tile
        const uint32_t xrow = sbase + slot * kStageBytes + warp * kSegBytes;
        __syncwarp();  // the previous row's T has been read by every lane
#pragma unroll
        for (int tp = 0; tp < 4; ++tp) {
          uint32_t x0, x1, x2, x3;  // tiles 2tp (x0, x1) and 2tp+1 (x2, x3)
          ldsm_x4(xrow + tp * 512 + lane * 16, x0, x1, x2, x3);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t a0 = h ? x2 : x0, a1 = h ? x3 : x1;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_16816(d, a0, a1, a0, a1, fa_hm0, fa_hm1);
            mma_1688(d, a0, a1, fa_lo);
            // rows c = 32tp + 16h + g and c + 8: block c/4, row i = c%4, columns 2*t4, 2*t4+1;
            // 16-byte unit (2i + t4/2) of block blk sits at unit ^ (blk % 8)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int c = 32 * tp + 16 * h + g + 8 * r;
              const int blk = c >> 2, i = c & 3;
              sts_v2(tbuf + blk * 128 + ((((i << 1) | (t4 >> 1)) ^ (blk & 7)) << 4) + ((t4 & 1) << 3),
                     d[2 * r], d[2 * r + 1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (kStages + slot));  // X row consumed
      if (row_ok && active) {
        if (kPerRowClip) {
          const int64_t ri = m * p.nb + b;
          r_lo = p.g_lo ? clip_ratio(p.g_lo[ri]) : 1.0f;
          r_hi = p.g_hi ? clip_ratio(p.g_hi[ri]) : 1.0f;
        }
        // ---- 3: T rows as column pairs, t2[i][qq] = {T[i][2qq], T[i][2qq+1]}
        uint64_t t2[4][4];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = lds_v4(tbuf + lane * 128 + ((u ^ (lane & 7)) << 4));
          t2[u >> 1][(u & 1) * 2] = pack2(__uint_as_float(v.x), __uint_as_float(v.y));
          t2[u >> 1][(u & 1) * 2 + 1] = pack2(__uint_as_float(v.z), __uint_as_float(v.w));
        }
        // ---- Y = B^T T  (Y[j][q] = sum_i B[i][j] T[i][q])
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
        // ---- block clip: [r_lo * min, r_hi * max]; 3-input min/max trees
        float tmn[11], tmx[11];
#pragma unroll
        for (int k = 0; k < 10; ++k) {
          tmn[k] = min3f(y[3 * k], y[3 * k + 1], y[3 * k + 2]);
          tmx[k] = max3f(y[3 * k], y[3 * k + 1], y[3 * k + 2]);
        }
        tmn[10] = fminf(y[30], y[31]);
        tmx[10] = fmaxf(y[30], y[31]);
        const float mn = fminf(min3f(min3f(tmn[0], tmn[1], tmn[2]), min3f(tmn[3], tmn[4], tmn[5]),
                                     min3f(tmn[6], tmn[7], tmn[8])),
                               fminf(tmn[9], tmn[10]));
        const float mx = fmaxf(max3f(max3f(tmx[0], tmx[1], tmx[2]), max3f(tmx[3], tmx[4], tmx[5]),
                                     max3f(tmx[6], tmx[7], tmx[8])),
                               fmaxf(tmx[9], tmx[10]));
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
