// Row quantizer on the CUDA cores and the KV-cache path of the BATQuant transformer
// integration (BATQuant note, en.papernotes.org, Method > Key Designs 4 "Equivalent
// Transformer integration": one transform set on the per-head key cache path and one
// on the value path; the KV8 / KV4 settings of Loss & Training store the cache in
// MXFP8 (E4M3) / MXFP4).
//
// bat_rows_quantize_kernel handles batches with few rows: decode-sized activations
// (its output is the tiled MXFP4 / MXFP8 layout the GEMM reads) and KV-cache stores,
// where every head's D-vector (D = head_dim, a multiple of 32) goes through the block
// transform y_b = x_b (B_b (x) A) with the same factors for all heads (A s x s shared,
// B_b (32/s) x (32/s) for each 32-channel block of the head), the block clip with
// per-block logits shared by heads and tokens, and MX quantization; the codes and
// the scale byte go to the token's cache slot. Larger batches go to the tensor-core
// prologue. bat_kv_dequantize_kernel reads cache rows back.
#pragma once

#include "bat_common.cuh"

namespace bat {

namespace kv {
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxBlocks = 8;     // D <= 256: P blocks staged in shared memory (32 KB)
constexpr int kFacFloats = 2112;  // A and B staged for the build when they fit (s >= 2)
}  // namespace kv


struct KvReadParams {
  const uint8_t* codes;   // cache codes
  const uint8_t* scales;  // cache scales [S][H][D/32]
  const int64_t* slots;   // [T]: cache rows to read
  const float* a;         // optional output factors (null: values as stored)
  const float* b;
  void* out;              // [T][H][D] fp32 or bf16
  int64_t T, H, S;
  int D, nbh, groups, ls;
};

// P_b[k][n] = B_b[k/s][n/s] * A[k%s][n%s] in fp32 for the head's nbh blocks. A and B
// are first copied to `fac` with coalesced loads when they fit (every split but s = 1,
// whose 32 x 32 private factors are read where they are). Ends with a CTA barrier.
__device__ __forceinline__ void kv_build_p(float* sp, float* fac, const float* a, const float* b,
                                           int nbh, int ls) {
  const int sm = (1 << ls) - 1, t = 32 >> ls;
  const int na = 1 << (2 * ls), nbf = nbh << (10 - 2 * ls);
  const bool staged = (na + 3) / 4 * 4 + nbf <= kv::kFacFloats;
  const float* sa = a;
  const float* sb = b;
  if (staged) {
    float* fb = fac + (na + 3) / 4 * 4;
    for (int i = threadIdx.x; i < na; i += blockDim.x) fac[i] = a[i];
    for (int i = threadIdx.x; i < nbf; i += blockDim.x) fb[i] = b[i];
    __syncthreads();
    sa = fac;
    sb = fb;
  }
  for (int i = threadIdx.x; i < nbh * 1024; i += blockDim.x) {
    const int blk = i >> 10, k = (i >> 5) & 31, n = i & 31;
    sp[i] = __fmul_rn(sb[(blk * t + (k >> ls)) * t + (n >> ls)], sa[((k & sm) << ls) + (n & sm)]);
  }
  __syncthreads();
}

// y[0..3] = outputs 4u..4u+3 of the lane's block: sum over k of x[k] * P[k][n],
// x[k] held by lane (l & ~7) + k/4 as its element k%4; k ascending.
__device__ __forceinline__ void kv_block_product(const float* pblk, const float (&x)[4], int lane,
                                                 float (&y)[4]) {
  const int base = lane & ~7, u = lane & 7;
  y[0] = y[1] = y[2] = y[3] = 0.0f;
#pragma unroll
  for (int src = 0; src < 8; ++src) {
    float xs[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xs[i] = __shfl_sync(0xffffffffu, x[i], base + src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 pr = *reinterpret_cast<const float4*>(pblk + (4 * src + i) * 32 + 4 * u);
      y[0] = __fmaf_rn(xs[i], pr.x, y[0]);
      y[1] = __fmaf_rn(xs[i], pr.y, y[1]);
      y[2] = __fmaf_rn(xs[i], pr.z, y[2]);
      y[3] = __fmaf_rn(xs[i], pr.w, y[3]);
    }
  }
}

// ---------------------------------------------------------------- row quantizer
// Small batches of rows (decode-sized activations, and KV-cache stores) on the CUDA
// cores: the tensor-core prologue's fixed costs (TMEM, barriers, the P_b build of a
// whole strip) dominate when there are few rows. Warp w always takes the same group
// g = w % groups of four 32-channel blocks, so lane l always works on block
// 4g + l/8 and keeps its four columns 4(l%8) .. 4(l%8)+3 of that block's P_b
// (32 x 4 fp32, the product B_b[k/s][n/s] * A[k%s][n%s] rounded once) and its clip
// ratios in registers; rows r0, r0 + R, ... of that group follow. Each row reads the
// block's 32 inputs directly (the block's eight lanes load the same 64 bytes) and
// sums x[k] * P_b[k][n] in fp32, k ascending.
struct RowQuantParams {
  const uint16_t* x;      // bf16 [rows][D]
  const float* a;         // [s][s]
  const float* b;         // [D/32][t][t]: one factor per 32-channel block of a row
  const float* g_lo;      // [D/32] clip logits, or null (no clip)
  const float* g_hi;
  uint8_t* codes;
  uint8_t* scales;
  float* y_out;           // optional fp32 [rows][D] trace of the transformed values
  const int64_t* slots;   // KV mode: cache slot of token row / H (-1 skips); else null
  int64_t rows;           // KV: tokens x heads; linear: M
  int64_t H;              // KV: heads per token (linear: 1)
  int64_t S;              // KV: cache slots
  int D, nb, groups, ls;  // D = channels per row, nb = D/32, groups = ceil(nb/4), log2 s
  int R;                  // warps per group: row stride
  int nbp4;               // linear mode: ceil(nb/4) of the tiled scale layout
  // optional completion flags (linear mode): CTA i stores `epoch` into done_flags[i]
  // (release, GPU scope) once all its outputs are written; null: none
  unsigned long long* done_flags;
  unsigned long long epoch;
};

// kKv: rows are (token, head) pairs stored into cache slots (codes [slot][H][D] or
// [slot][H][D/2], scales plain [slot][H][D/32]); otherwise rows of an activation
// matrix (codes [M][D] or [M][D/2], scales in the GEMM's tiled layout, padding 0).
template <bool kFp8, bool kTrace, bool kKv>
__global__ void __launch_bounds__(kv::kThreads, 1)
    bat_rows_quantize_kernel(const RowQuantParams p) {
  // per warp (factor split s = 8): A, the group's four B_b, its four pairs of clip logits
  __shared__ float fac_smem[kv::kWarps][136];
  // a following kernel launched with programmatic serialization (the GEMM) may start
  // its set-up now; this kernel's inputs come from the kernels before it
  allow_dependents();
  grid_dependency_wait();
  if (!kKv) {
    // padding of the tiled scale layout: rows [M, 128-row boundary) and blocks
    // [nb, 4 nbp4) of the real rows are 0 (the GEMM multiplies by 2^(byte-127)); done
    // first, so these stores overlap the loads below
    const int64_t mpad = (p.rows + 127) / 128 * 128;
    const int64_t tail = 4 * p.nbp4 - p.nb;  // 0..3 padding blocks per real row
    const int64_t n_rows_pad = (mpad - p.rows) * p.nbp4;
    const int64_t total = n_rows_pad + p.rows * tail;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      if (i < n_rows_pad) {
        const int64_t m = p.rows + i / p.nbp4;
        const int64_t c = i % p.nbp4;
        *reinterpret_cast<uint32_t*>(p.scales + scale_offset(m, 4 * c, p.nbp4)) = 0u;
      } else {
        const int64_t j = i - n_rows_pad;
        p.scales[scale_offset(j / tail, p.nb + j % tail, p.nbp4)] = 0;
      }
    }
  }
  const int lane = threadIdx.x & 31;
  const int u = lane & 7;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * kv::kWarps + (threadIdx.x >> 5);
  if (wid < static_cast<int64_t>(p.groups) * p.R) {
    const int g = static_cast<int>(wid % p.groups);
    const int blk = 4 * g + (lane >> 3);
    const bool has = blk < p.nb;  // lanes of a missing fourth block idle (shuffles stay full)
    const int bq = has ? blk : 0;
    // the first row's block is requested before the factors, so that its load and theirs
    // are in flight together
    int64_t row = wid / p.groups;
    float x[32];
    if (row < p.rows) rows_load_block(p.x + row * p.D + bq * kG, x);
    float r_lo = 1.0f, r_hi = 1.0f;
    float pc[32][4];
    if (p.ls == 3) {
      // A (8 x 8), the four blocks' B_b (4 x 4 each) and clip logits: one load per lane
      // or two, all in flight at once, into this warp's shared-memory slice
      float* f = fac_smem[threadIdx.x >> 5];
      const int b0 = 4 * g;
      f[lane] = __ldg(p.a + lane);
      f[32 + lane] = __ldg(p.a + 32 + lane);
      if (b0 + (lane >> 4) < p.nb) f[64 + lane] = __ldg(p.b + b0 * 16 + lane);
      if (b0 + 2 + (lane >> 4) < p.nb) f[96 + lane] = __ldg(p.b + b0 * 16 + 32 + lane);
      if (lane < 4 && b0 + lane < p.nb) {
        f[128 + lane] = p.g_lo ? __ldg(p.g_lo + b0 + lane) : 0.0f;
        f[132 + lane] = p.g_hi ? __ldg(p.g_hi + b0 + lane) : 0.0f;
      }
      __syncwarp();
      const int bl = has ? blk - b0 : 0;  // the lane's block within the four
      if (has && p.g_lo) r_lo = clip_ratio(f[128 + bl]);
      if (has && p.g_hi) r_hi = clip_ratio(f[132 + bl]);
      rows_build_pc<3, false>(pc, f, f + 64, bl, u, 3);
    } else {
      if (has && p.g_lo) r_lo = clip_ratio(p.g_lo[bq]);
      if (has && p.g_hi) r_hi = clip_ratio(p.g_hi[bq]);
      rows_build_pc<-1>(pc, p.a, p.b, bq, u, p.ls);
    }
    for (; row < p.rows; row += p.R) {
      int64_t slot = row;
      if (kKv) {
        slot = p.slots[row / p.H];
        if (slot >= p.S) {
          if (lane == 0) atomicOr(&g_dev_error, kErrBadIndex);
          if (row + p.R < p.rows) rows_load_block(p.x + (row + p.R) * p.D + bq * kG, x);
          continue;
        }
      }
      float y[4];
      uint32_t code;
      int sbyte;
      rows_block_quant<kFp8>(x, pc, r_lo, r_hi, y, code, sbyte);
      // the next row's block (this one's values are consumed)
      if (row + p.R < p.rows) rows_load_block(p.x + (row + p.R) * p.D + bq * kG, x);
      const int64_t e0 = row * p.D + blk * kG + 4 * u;
      if (kTrace && has)
        *reinterpret_cast<float4*>(p.y_out + e0) = make_float4(y[0], y[1], y[2], y[3]);
      if (!has || slot < 0) continue;
      // element index of the code: cache row (slot, head) or the activation row
      const int64_t crow = kKv ? slot * p.H + row % p.H : row;
      const int64_t ci = crow * p.D + blk * kG + 4 * u;
      if (kFp8)
        *reinterpret_cast<uint32_t*>(p.codes + ci) = code;
      else
        *reinterpret_cast<uint16_t*>(p.codes + ci / 2) = static_cast<uint16_t>(code);
      if (u == 0) {
        if (kKv)
          p.scales[crow * p.nb + blk] = static_cast<uint8_t>(sbyte);
        else
          p.scales[scale_offset(row, blk, p.nbp4)] = static_cast<uint8_t>(sbyte);
      }
    }
  }
  if (!kKv && p.done_flags != nullptr) {
    // every thread of the CTA has written its outputs; thread 0 publishes them (the
    // barrier orders the others' stores before its release)
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      st_release_gpu_u64(p.done_flags + blockIdx.x, p.epoch);
    }
  }
}

// E4M3 / E2M1 code -> value (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if ((c & 0x7Fu) == 0x7Fu) return __uint_as_float(0x7FC00000u);
  const float mag = e == 0 ? static_cast<float>(m) * 0x1p-9f
                           : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80u) ? -mag : mag;
}
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t i = c & 7u;
  // 0, 0.5, 1, 1.5 (i < 4) then 2, 3, 4, 6
  const float mag = i < 4 ? 0.5f * static_cast<float>(i) : static_cast<float>((i & 1 ? 3 : 2) << ((i - 4) >> 1));
  return (c & 8u) ? -mag : mag;
}

template <bool kFp8, bool kXform, bool kF32Out>
__global__ void __launch_bounds__(kv::kThreads)
    bat_kv_dequantize_kernel(const KvReadParams p) {
  __shared__ __align__(16) float sp[kXform ? kv::kMaxBlocks * 1024 : 4];
  __shared__ __align__(16) float fac[kXform ? kv::kFacFloats : 4];
  if (kXform) kv_build_p(sp, fac, p.a, p.b, p.nbh, p.ls);
  const int lane = threadIdx.x & 31;
  const int u = lane & 7;
  const int64_t items = p.T * p.H * p.groups;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kv::kWarps;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * kv::kWarps + (threadIdx.x >> 5); it < items;
       it += wstride) {
    const int g = static_cast<int>(it % p.groups);
    const int64_t th = it / p.groups;
    const int64_t t = th / p.H;
    const int blk = 4 * g + (lane >> 3);
    const bool has = blk < p.nbh;
    const int64_t slot = p.slots[t];
    const bool ok = slot >= 0 && slot < p.S;
    if (!ok && lane == 0) atomicOr(&g_dev_error, kErrBadIndex);
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (has && ok) {
      const int64_t crow = (slot * p.H + th % p.H) * p.D + blk * kG + 4 * u;
      const uint32_t sb = p.scales[(slot * p.H + th % p.H) * p.nbh + blk];
      const float sc = sb == 255u ? __uint_as_float(0x7FC00000u)
                                  : (sb == 0u ? 0x1p-127f : __uint_as_float(sb << 23));
      if (kFp8) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p.codes + crow);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = e4m3_value((w >> (8 * i)) & 0xFFu) * sc;
      } else {
        const uint32_t w = *reinterpret_cast<const uint16_t*>(p.codes + crow / 2);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = e2m1_value((w >> (4 * i)) & 0xFu) * sc;
      }
    }
    float y[4] = {v[0], v[1], v[2], v[3]};
    if (kXform) kv_block_product(sp + (has ? blk : 0) * 1024, v, lane, y);
    if (!has) continue;
    const int64_t e0 = th * p.D + blk * kG + 4 * u;
    if (kF32Out) {
      *reinterpret_cast<float4*>(static_cast<float*>(p.out) + e0) = make_float4(y[0], y[1], y[2], y[3]);
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(y[0], y[1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(y[2], y[3]);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + e0) = w;
    }
  }
}

}  // namespace bat
