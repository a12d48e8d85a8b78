// Fused prologue: GPK block transform + block-wise clipping + MXFP4 quantize/pack.
//
// BATQuant note (en.papernotes.org), Method > Key Designs 2 and 3: each
// 32-channel block x (a row-major 4x8 matrix X_r) becomes
// y = vec_row(B_b^T X_r A) — two small matrix products instead of the explicit
// 32x32 block B_b (x) A — then is clipped to [r_lo*min(y), r_hi*max(y)] and
// quantized to E2M1 codes with one UE8M0 scale 2^e, e = floor(log2 amax) - 2.
//
// Work mapping: one lane owns one 32-element block. A warp covers 32
// consecutive blocks of one row (2 KB of bf16, read as 64 contiguous bytes per
// lane), so the shared factor A (64 fp32) stays in registers for the whole
// kernel and the private factor B_b is reloaded only when the lane's block
// changes. The transform runs on packed fp32x2 FMAs. The block min/max, clip
// bounds, scale and codes never leave registers; each lane writes its 16 bytes
// of codes with one vector store and its scale byte into the tiled order the
// GEMM reads.
#pragma once

#include "bat_common.cuh"

namespace bat {

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
};

// fp32(sigma(g)) evaluated in fp64; +inf gives exactly 1.
__device__ __forceinline__ float clip_ratio(float g) {
  if (isinf(g) && g > 0.0f) return 1.0f;
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(g))));
}

__device__ __forceinline__ int64_t scale_offset(int64_t m, int64_t b, int nbp4) {
  return ((m >> 7) * nbp4 + (b >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (b & 3);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// kPerRowClip: clip logits indexed [row][block] (weight side) instead of [block].
template <bool kTrace, bool kPerRowClip>
__global__ void __launch_bounds__(256) bat_prologue_kernel(const PrologueParams p) {
  extern __shared__ float s_ratio[];  // [2][nb] when !kPerRowClip
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nb = p.nb;

  if (!kPerRowClip) {
    for (int t = threadIdx.x; t < nb; t += blockDim.x) {
      s_ratio[t] = p.g_lo ? clip_ratio(p.g_lo[t]) : 1.0f;
      s_ratio[nb + t] = p.g_hi ? clip_ratio(p.g_hi[t]) : 1.0f;
    }
    __syncthreads();
  }

  // Shared factor A as packed column pairs: a2[p][qq] = {A[p][2qq], A[p][2qq+1]}.
  uint64_t a2[8][4];
#pragma unroll
  for (int pp = 0; pp < 8; ++pp)
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const float2 v = reinterpret_cast<const float2*>(p.a)[pp * 4 + qq];
      a2[pp][qq] = pack2(v.x, v.y);
    }

  const int64_t units = p.rows * p.nseg;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  int cur_b = -1;
  uint64_t b2[4][4];  // b2[i][j] = {B[i][j], B[i][j]}
  float r_lo = 1.0f, r_hi = 1.0f;

  for (int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; u < units;
       u += wstride) {
    const int seg = static_cast<int>(u / p.rows);
    const int64_t m = u - static_cast<int64_t>(seg) * p.rows;
    const int b = seg * 32 + lane;
    if (b >= nb) continue;
    if (b != cur_b) {
      cur_b = b;
      const float4* bp = reinterpret_cast<const float4*>(p.b + static_cast<int64_t>(b) * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(bp + i);
        b2[i][0] = pack2(v.x, v.x);
        b2[i][1] = pack2(v.y, v.y);
        b2[i][2] = pack2(v.z, v.z);
        b2[i][3] = pack2(v.w, v.w);
      }
      if (!kPerRowClip) {
        r_lo = s_ratio[b];
        r_hi = s_ratio[nb + b];
      }
    }
    if (kPerRowClip) {
      const int64_t ri = m * nb + b;
      r_lo = p.g_lo ? clip_ratio(p.g_lo[ri]) : 1.0f;
      r_hi = p.g_hi ? clip_ratio(p.g_hi[ri]) : 1.0f;
    }

    // ---- load the block: 32 bf16 = 64 bytes
    const uint16_t* src = p.x + m * p.K + static_cast<int64_t>(b) * kG;
    uint32_t w[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = ldg_nc_v4(src + 8 * c);
      w[4 * c + 0] = v.x;
      w[4 * c + 1] = v.y;
      w[4 * c + 2] = v.z;
      w[4 * c + 3] = v.w;
    }

    // ---- T = X_r A  (X_r[i][p] = x[8i+p]; word 4i + p/2 holds x[8i+p], p even in the low half)
    uint64_t t2[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) t2[i][qq] = 0ull;
#pragma unroll
      for (int pp = 0; pp < 8; ++pp) {
        const uint32_t word = w[4 * i + (pp >> 1)];
        const float xv = (pp & 1) ? bf16hi(word) : bf16lo(word);
        const uint64_t xx = pack2(xv, xv);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) t2[i][qq] = ffma2(xx, a2[pp][qq], t2[i][qq]);
      }
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

    if (kTrace) {
      float4* dst = reinterpret_cast<float4*>(p.y_out + m * p.K + static_cast<int64_t>(b) * kG);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
    }

    // ---- block clip: [r_lo * min, r_hi * max]
    float mn = y[0], mx = y[0];
#pragma unroll
    for (int k = 1; k < 32; ++k) {
      mn = fminf(mn, y[k]);
      mx = fmaxf(mx, y[k]);
    }
    const float lo = __fmul_rn(r_lo, mn);
    const float hi = __fmul_rn(r_hi, mx);
    // The clamp is monotone, so the clipped block's extremes are the clipped min/max.
    const float amax =
        fmaxf(fabsf(fminf(fmaxf(mn, lo), hi)), fabsf(fminf(fmaxf(mx, lo), hi)));

    // ---- UE8M0 scale: e = floor(log2 amax) - 2, clamped to >= -127 (amax = 0 -> -127)
    const int efield = static_cast<int>(__float_as_uint(amax) >> 23);
    const int sbyte = efield > 2 ? efield - 2 : 0;            // e + 127
    const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);  // 2^-e
    const uint64_t s2 = pack2(inv_scale, inv_scale);

    // ---- codes: v = c * 2^-e (+0 turns an exact -0 into +0), E2M1 round-to-nearest-even
    uint32_t packed[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t word = 0;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int k = 8 * c + 2 * h;
        const float c0 = fminf(fmaxf(y[k], lo), hi);
        const float c1 = fminf(fmaxf(y[k + 1], lo), hi);
        float v0, v1;
        unpack2(ffma2(pack2(c0, c1), s2, 0ull), v0, v1);
        word |= e2m1x2(v0, v1) << (8 * h);
      }
      packed[c] = word;
    }
    uint4* cdst = reinterpret_cast<uint4*>(p.codes + (m * p.K + static_cast<int64_t>(b) * kG) / 2);
    *cdst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    p.scales[scale_offset(m, b, p.nbp4)] = static_cast<uint8_t>(sbyte);
  }

  // ---- zero the padding bytes of the tiled scale buffer
  const int64_t rows_pad = (p.rows + 127) & ~static_cast<int64_t>(127);
  const int64_t bcols = static_cast<int64_t>(p.nbp4) * 4;
  const int64_t pad_cols = bcols - nb;                 // blocks past nb, rows < M
  const int64_t n_right = p.rows * pad_cols;
  const int64_t n_below = (rows_pad - p.rows) * bcols; // rows past M, all blocks
  const int64_t tstride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       t < n_right + n_below; t += tstride) {
    int64_t m, b;
    if (t < n_right) {
      m = t / pad_cols;
      b = nb + (t - m * pad_cols);
    } else {
      const int64_t r = t - n_right;
      m = p.rows + r / bcols;
      b = r - (m - p.rows) * bcols;
    }
    p.scales[scale_offset(m, b, p.nbp4)] = 0;
  }
}

__global__ void bat_clip_ratio_kernel(const float* g, int64_t n, float* r) {
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    r[t] = g ? clip_ratio(g[t]) : 1.0f;
}

}  // namespace bat
