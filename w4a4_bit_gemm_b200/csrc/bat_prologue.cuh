// Fused prologue: GPK block transform + block-wise clipping + MXFP4 quantize/pack.
//
// BATQuant note (en.papernotes.org), Method > Key Designs 2 and 3: each
// 32-channel block x of a token becomes y = x (B_b (x) A) = vec_row(B_b^T X_r A),
// then is clipped to [r_lo*min(y), r_hi*max(y)] and quantized to E2M1 codes with
// one UE8M0 scale 2^e, e = floor(log2 amax) - 2.
//
// All tokens share the 32x32 matrix P_b = B_b (x) A of block column b, so the
// transform of 128 tokens is one dense product X_b (128x32) . P_b (32x32): a
// 5th-generation tensor-core MMA (tcgen05, kind::f16, bf16 operands, fp32
// accumulators in TMEM). x is exact in bf16; P_b (each entry the fp32 product
// B_b[i][j] * A[p][q]) is split into three bf16 terms P_hi + P_mid + P_lo
// (residual ~2^-24 |P_b|). The three terms sit side by side as one N=96 operand,
// so one MMA per 16-wide K-step reads the X tile once and yields the three
// partial products, which the quantizer adds in fp32: y matches an fp32 product
// to within fp32 rounding. The accumulator puts token m in TMEM lane m, so a
// thread holds the whole 32-element block of one token: block min/max, clip,
// scale and E2M1 codes need no exchange between threads.
//
// Work unit: 128 tokens x one pair of blocks (a 128-row x 128-byte box of X).
// Block pairs are grouped into strips of kStrip pairs; each CTA owns one strip
// (the P terms of all its blocks stay in shared memory) and a contiguous range
// of its units, walked token tile by token tile with the strip's pairs inner, so
// that consecutive copies read adjacent 128-byte pieces of the same 128 rows.
//   warp 0      producer: TMA copies of the units' boxes into a ring of kStages
//               shared-memory stages;
//   warps 1, 18 MMA issuers, taking alternate units (unit n uses accumulator n % 2):
//               per unit, two blocks x two K-steps of M=128, N=96, K=16 into one of
//               two 192-column accumulators. The issuing thread waits about 150
//               cycles on each MMA (the tensor pipe takes one M=128, K=16 step at a
//               time) and some 100 on each barrier wait and commit, so with one issuer
//               the tensor pipe idles while it waits; with two, one issues while the
//               other waits. Warp 1 also owns TMEM;
//   warps 2-17  two quantizer sets of eight warps; set s takes the units whose
//               index within the CTA is s mod 2, warp (s, j, q) block j of the
//               pair for the 32 tokens of TMEM lane quarter q.
// Warps 1-18 build the strip's P terms (and its blocks' clip ratios) while the
// producer's first copies are in flight. The issuer waits once per unit for its
// copy and once for its accumulator, so its chain of waits, MMAs and commits
// stays inside the copy's time, and each quantizer set has two units' time for
// one block.
#pragma once

#include "bat_common.cuh"

namespace bat {

namespace pro {
constexpr int kTok = 128;                        // tokens per unit (MMA M)
constexpr int kBlk = 2;                          // 32-element blocks per unit
constexpr int kStrip = 4;                        // block pairs per strip
constexpr int kStages = 10;
constexpr int kStageBytes = kTok * 128;          // 128 rows x 64 bf16: 16 KB
constexpr int kPTermBytes = 32 * 32 * 2;         // one bf16 term of one block's P: 2 KB
constexpr int kPBlockBytes = 3 * kPTermBytes;    // one block's three terms: 6 KB
constexpr int kPPairBytes = kBlk * kPBlockBytes; // 12 KB
constexpr int kPBytes = kStrip * kPPairBytes;    // one strip: 48 KB
constexpr int kSets = 2;                         // quantizer sets (alternate units)
constexpr int kSetWarps = 4 * kBlk;              // lane quarters x blocks
constexpr int kIssuers = 2;                      // MMA issuer warps (alternate units)
constexpr int kThreads = 32 * (1 + kIssuers + kSets * kSetWarps);
constexpr int kBuilders = kThreads - 32;         // every warp but the producer
constexpr int kBarBytes = 2048;                  // barriers, TMEM address, clip ratios
// A and the strip's B_b staged for the P build: s*s + 2*kStrip*(32/s)^2 floats, at most
// 2052 (s = 2); the fully private split (s = 1, 8193 floats) reads them from global memory
constexpr int kFacFloats = 2112;
constexpr bool fac_fits(int ls) {
  return ls > 5 || (((1 << (2 * ls)) + 3) / 4 * 4 + 2 * kStrip * (1 << (10 - 2 * ls)) <= kFacFloats &&
                    fac_fits(ls + 1));
}
static_assert(fac_fits(1), "the staged factors of every split s >= 2 fit the staging area");
constexpr int kSmemBytes = kStages * kStageBytes + kPBytes + kBarBytes + 4 * kFacFloats + 1024;
static_assert(kStages % kIssuers == 0 && kIssuers == 2, "issuer i owns accumulator i and every other stage");
constexpr int kSlotCols = 96;                    // one block's accumulator: 3 terms x 32 columns
constexpr uint32_t kAccCols = kBlk * kSlotCols;  // one unit's accumulator: 192 columns
constexpr uint32_t kTmemCols = 512;              // allocation (power of two) holding 2 x 192
}  // namespace pro

struct PrologueParams {
  const float* a;        // fp32 [s][s], shared factor (s = 1 << ls)
  const float* b;        // fp32 [nb][32/s][32/s], private factors
  const float* g_lo;     // clip logits: [nb] (shared by rows) or [rows][nb]; may be null
  const float* g_hi;
  uint8_t* codes;        // [rows][K/2] packed E2M1, or [rows][K] E4M3 (kFp8)
  uint8_t* scales;       // tiled, rows padded to 128, blocks padded to 4
  float* y_out;          // optional fp32 [rows][K] trace of the transformed values
  int64_t rows;
  int64_t K;
  int nb;                // K / 32
  int nbp2;              // ceil(nb / 2): block pairs
  int nbp4;              // ceil(nb / 4): groups of the tiled scale layout
  int64_t mtiles;        // ceil(rows / 128)
  int strips;            // ceil(nbp2 / kStrip)
  int cps;               // CTAs per strip (grid = strips * cps)
  int ls;                // log2 of the shared factor's size: 0..5 (3 is the 8 x 8 / 4 x 4 split)
  // KV-cache store (kKv): row m = token (m / kv_heads), head (m % kv_heads); its codes go
  // to cache row slots[token] * kv_heads + head, scales plain [cache row][nb]
  const int64_t* slots;
  int64_t kv_heads;
  int64_t kv_slots;
  // optional completion flags (linear mode): CTA i stores `epoch` into cta_flags[i]
  // (release, GPU scope) once all its codes and scales are written; null: none. (CTA i
  // covers strip i / cps, units [sunits (i % cps) / cps, sunits (i % cps + 1) / cps).)
  unsigned long long* cta_flags;
  unsigned long long epoch;
};




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

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major), fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
  return 1u << 4 |                                 // D format: fp32
         1u << 7 |                                 // A format: bf16
         1u << 10 |                                // B format: bf16
         static_cast<uint32_t>(n >> 3) << 17 |     // N / 8
         static_cast<uint32_t>(m >> 4) << 24;      // M / 16
}
// D[tmem] (+)= A x B^T, bf16 operands from shared memory, M=128, K=16.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The three bf16 terms of P_b for block b, in the MMA's B-operand layout (N x K,
// K-major, no swizzle: 8x8 core matrices of 128 bytes, K-adjacent ones 128 bytes
// apart, N-adjacent ones 512 bytes apart; the terms follow one another, so the
// three together are one N=96 operand). With A of size s x s (s = 1 << ls) and
// B_b of size t x t (t = 32 / s), operand element (n, k) is
// P_b[k][n] = B_b[k/s][n/s] * A[k%s][n%s], rounded once to fp32 and split
// exactly into three bf16 terms. `row` in [0, 128) picks n = row/4 and the eight
// k of core-matrix column row%4: one 16-byte row of a core matrix per term.
// `a` and `bb` point at A and B_b, staged in shared memory or in global memory;
// `bb` is null for a block past nb, which gets 0.
__device__ __forceinline__ void build_p_row(uint8_t* dst, const float* a, const float* bb, int ls,
                                            int row) {
  const int n = row >> 2, kc = row & 3;
  const int sm = (1 << ls) - 1, t = 32 >> ls;
  const int an = n & sm, bn = n >> ls;
  uint32_t w[3][4];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    uint32_t hh[2], mm[2], ll[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = kc * 8 + i + h;
      const float bv = bb ? bb[(k >> ls) * t + bn] : 0.0f;
      const float prod = __fmul_rn(bv, a[((k & sm) << ls) + an]);
      const uint32_t hi = bf16_bits(prod);
      const float r1 = prod - __uint_as_float(hi << 16);
      const uint32_t mid = bf16_bits(r1);
      hh[h] = hi;
      mm[h] = mid;
      ll[h] = bf16_bits(r1 - __uint_as_float(mid << 16));
    }
    w[0][i >> 1] = hh[0] | (hh[1] << 16);
    w[1][i >> 1] = mm[0] | (mm[1] << 16);
    w[2][i >> 1] = ll[0] | (ll[1] << 16);
  }
  const int off = ((n >> 3) * 4 + kc) * 128 + (n & 7) * 16;
#pragma unroll
  for (int term = 0; term < 3; ++term)
    *reinterpret_cast<uint4*>(dst + term * pro::kPTermBytes + off) =
        make_uint4(w[term][0], w[term][1], w[term][2], w[term][3]);
}

// Quantize one 32-element block held by this thread: clip to [r_lo*min, r_hi*max],
// UE8M0 scale, then E2M1 codes (MXFP4: 16 bytes into `packed`) or, with kFp8, OCP
// E4M3 codes (MXFP8: 32 bytes). Returns the scale byte e + 127.
//
// The clip is applied to the codes rather than to the values. The conversion is
// monotone and symmetric, so the code of a clamped value is the code of the unclamped
// value with its magnitude capped at the magnitude code of the bound on its side:
// hi for a positive value, min(lo, hi) for a negative one (lo > hi happens only in a
// one-signed block, where every value ends at hi). Codes are sign-magnitude with the
// magnitude's order that of the values, so the cap is an unsigned minimum per code,
// done on 8 packed E2M1 codes (or 4 E4M3 codes) per 32-bit word with integer ops.
// This gives the codes of the value-domain clip exactly (the bound values are
// converted the same way, fma(bound, 2^-e, +0)), with half the per-element work.
template <int kBits>  // 4: E2M1 nibbles, 8: E4M3 bytes
__device__ __forceinline__ uint32_t cap_codes(uint32_t w, uint32_t bp, uint32_t bn) {
  constexpr uint32_t kOnes = kBits == 4 ? 0x11111111u : 0x01010101u;
  constexpr uint32_t kSign = kOnes << (kBits - 1);       // sign bit of every code
  constexpr uint32_t kMagMax = (1u << (kBits - 1)) - 1;  // 7 or 0x7f
  const uint32_t neg = (w >> (kBits - 1)) & kOnes;       // 1 per negative code
  const uint32_t bp_all = bp * kOnes, bn_all = bn * kOnes;
  const uint32_t bw = bp_all ^ ((bp_all ^ bn_all) & (neg * ((1u << kBits) - 1)));  // cap per code
  // per code: (sign bit set | magnitude) - cap >= sign bit  <=>  magnitude >= cap
  const uint32_t d = (w | kSign) - bw;
  const uint32_t sel = ((d >> (kBits - 1)) & kOnes) * kMagMax;
  return (w & ~sel) | (bw & sel);
}

template <bool kFp8>
__device__ __forceinline__ uint32_t quantize_block(const float (&y)[32], float r_lo, float r_hi,
                                                   uint32_t (&packed)[kFp8 ? 8 : 4]) {
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
  // UE8M0 scale: e = floor(log2 amax) - emax, with emax 2 (E2M1) or 8 (E4M3), clamped
  // to >= -127 (amax = 0 -> -127)
  constexpr int kEmax = kFp8 ? 8 : 2;
  const int efield = static_cast<int>(__float_as_uint(amax) >> 23);
  const int sbyte = efield > kEmax ? efield - kEmax : 0;  // e + 127
  const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);  // 2^-e
  const uint64_t s2 = pack2(inv_scale, inv_scale);
  // magnitude caps: codes of the bounds scaled the same way
  const float cap_p = __fmaf_rn(hi, inv_scale, 0.0f);
  const float cap_n = __fmaf_rn(fabsf(fminf(lo, hi)), inv_scale, 0.0f);
  // codes of the unclipped values v = y * 2^-e (+0 turns an exact -0 into +0), round to
  // nearest even, then capped
  if constexpr (kFp8) {
    const uint32_t caps = e4m3x4(cap_p, cap_n, 0.0f, 0.0f);
    const uint32_t bp = caps & 0x7fu, bn = (caps >> 8) & 0x7fu;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v[4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        unpack2(ffma2(pack2(y[4 * c + 2 * h], y[4 * c + 2 * h + 1]), s2, 0ull), v[2 * h], v[2 * h + 1]);
      packed[c] = cap_codes<8>(e4m3x4(v[0], v[1], v[2], v[3]), bp, bn);
    }
  } else {
    const uint32_t caps = e2m1x2(cap_p, cap_n);
    const uint32_t bp = caps & 7u, bn = (caps >> 4) & 7u;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[8];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        unpack2(ffma2(pack2(y[8 * c + 2 * h], y[8 * c + 2 * h + 1]), s2, 0ull), v[2 * h], v[2 * h + 1]);
      packed[c] = cap_codes<4>(e2m1x8(v), bp, bn);
    }
  }
  return static_cast<uint32_t>(sbyte);
}

// tmap_x: bf16 X [rows][K], box 64 columns x 128 rows, 128-byte swizzle, zero fill.
// kPerRowClip: clip logits indexed [row][block] (weight side) instead of [block].
// kFp8: MXFP8 (E4M3) codes, one byte per element, instead of packed MXFP4.
// kKv: rows are (token, head) pairs of a K or V batch, stored into cache slots.
template <bool kTrace, bool kPerRowClip, bool kFp8 = false, bool kKv = false>
__global__ void __launch_bounds__(pro::kThreads, 1)
    bat_prologue_kernel(const __grid_constant__ CUtensorMap tmap_x, const PrologueParams p) {
  using namespace pro;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;  // 128-byte swizzle atoms: 1 KB aligned
  uint8_t* base_ptr = smem_raw + (base - raw_u32);
  const uint32_t pbase = base + kStages * kStageBytes;  // [pair][block][term][2 KB]
  uint8_t* pbase_ptr = base_ptr + kStages * kStageBytes;
  const uint32_t bars = pbase + kPBytes;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
  auto tfull = [&](uint32_t a) { return bars + 8u * (2 * kStages + a); };
  auto tempty = [&](uint32_t a) { return bars + 8u * (2 * kStages + 2 + a); };
  const uint32_t pfull = bars + 8u * (2 * kStages + 4);
  auto done_bar = [&](int i) { return pfull + 8u * (1 + i); };
  const uint32_t tmem_slot = pfull + 8u * (1 + kIssuers);
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(base_ptr + (tmem_slot - base));
  // clip ratios of the strip's blocks: [2 * kStrip] lo, then [2 * kStrip] hi
  float* ratios = reinterpret_cast<float*>(base_ptr + (bars - base) + 256);

  // A and the strip's B_b, staged for the P build (s > 1): A [s][s], then [2 * kStrip][t][t]
  const bool staged = p.ls > 0;
  const int fa = 1 << (2 * p.ls), fb = 1 << (10 - 2 * p.ls);  // s*s and t*t
  float* sA = reinterpret_cast<float*>(base_ptr + (bars - base) + kBarBytes);
  float* sB = sA + ((fa + 3) & ~3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // this CTA's strip and its contiguous range of the strip's units, unit v of the
  // strip = (token tile v / npair, pair strip * kStrip + v % npair)
  const int strip = static_cast<int>(blockIdx.x) / p.cps;
  const int part = static_cast<int>(blockIdx.x) - strip * p.cps;
  const int pair_base = strip * kStrip;
  const int npair = min(kStrip, p.nbp2 - pair_base);
  const int64_t sunits = p.mtiles * npair;
  const int64_t v_begin = sunits * part / p.cps;
  const int64_t v_end = sunits * (part + 1) / p.cps;
  const int64_t mt0 = v_begin / npair;
  const int pr0 = static_cast<int>(v_begin - mt0 * npair);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (uint32_t a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), kSetWarps);
    }
    mbar_init(pfull, kBuilders);
    for (int i = 0; i < kIssuers; ++i) mbar_init(done_bar(i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmap_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  // The next kernel on the stream (normally the GEMM) may start its own set-up now;
  // it waits for this grid to finish before it reads the codes.
  allow_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The boxes of one token tile (the strip's pairs, adjacent 128-byte pieces of
    // the same 128 rows) are issued back to back once enough stages are free, so
    // that the memory system sees whole row segments rather than lone 128-byte
    // pieces of rows 8 KB apart.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();  // X is read once
      int stage = 0;
      uint32_t phase = 0;
      uint32_t inflight = 0;  // bit s: stage s was loaded; bit 16+s: parity of that load
      int64_t mt = mt0;
      int pr = pr0;
      bool ok = true;
      for (int64_t v = v_begin; v < v_end && ok;) {
        int64_t cnt = npair - pr;
        if (cnt > v_end - v) cnt = v_end - v;
        if (cnt > kStages) cnt = kStages;
        // wait for the next cnt stages to be free
        int s2 = stage;
        uint32_t ph2 = phase;
        for (int i = 0; i < cnt; ++i) {
          if (!mbar_wait(empty_bar(s2), ph2 ^ 1u, kErrWaitEmpty)) { ok = false; break; }
          if (++s2 == kStages) { s2 = 0; ph2 ^= 1u; }
        }
        for (int i = 0; i < cnt && ok; ++i) {
          mbar_expect_tx(full_bar(stage), kStageBytes);
          tma_load_2d_hint(base + stage * kStageBytes, &tmap_x, full_bar(stage),
                           (pair_base + pr) * 64, static_cast<int32_t>(mt * kTok), pol);
          inflight = (inflight & ~(0x10001u << stage)) | (1u << stage) | (phase << (16 + stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
          if (++pr == npair) { pr = 0; ++mt; }
          ++v;
        }
      }
      // no copy may still be writing shared memory when the CTA exits
      for (int s = 0; s < kStages; ++s)
        if ((inflight >> s) & 1u) mbar_wait(full_bar(s), (inflight >> (16 + s)) & 1u, kErrWaitFull);
    }
  } else {
    // ------------------------------------------------ P terms and clip ratios
    {
      const int t = threadIdx.x - 32;
      // stage A and the strip's B_b with coalesced loads (zeros for blocks past nb)
      if (staged) {
        for (int i = t; i < fa; i += kBuilders) sA[i] = p.a[i];
        const int64_t e0 = 2 * static_cast<int64_t>(pair_base) * fb;
        const int64_t e_end = static_cast<int64_t>(p.nb) * fb;
        for (int i = t; i < 2 * npair * fb; i += kBuilders) sB[i] = e0 + i < e_end ? p.b[e0 + i] : 0.0f;
      }
      if (!kPerRowClip && t >= 320 && t < 320 + 2 * npair) {
        const int lb = t - 320;
        const int64_t blk = 2 * static_cast<int64_t>(pair_base) + lb;
        const bool ok = blk < p.nb;
        ratios[lb] = (ok && p.g_lo) ? clip_ratio(p.g_lo[blk]) : 1.0f;
        ratios[2 * kStrip + lb] = (ok && p.g_hi) ? clip_ratio(p.g_hi[blk]) : 1.0f;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kBuilders) : "memory");  // warps 1-17
      // pairs this CTA's units touch: all of the strip's, or a short run of them
      const int64_t nv = v_end - v_begin;
      for (int r = t; r < npair * 2 * 128; r += kBuilders) {
        const int pr = r >> 8, jj = (r >> 7) & 1;
        const bool used = nv >= npair || ((pr - pr0 + npair) % npair) < nv;
        if (!used) continue;
        uint8_t* dst = pbase_ptr + pr * kPPairBytes + jj * kPBlockBytes;
        if (p.ls == 3) {  // the default split, with its shifts folded into constants
          build_p_row(dst, sA, sB + (2 * pr + jj) * 16, 3, r & 127);
        } else if (staged) {
          build_p_row(dst, sA, sB + (2 * pr + jj) * fb, p.ls, r & 127);
        } else {
          const int blk = 2 * (pair_base + pr) + jj;
          build_p_row(dst, p.a, blk < p.nb ? p.b + static_cast<int64_t>(blk) * fb : nullptr, p.ls,
                      r & 127);
        }
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor cores
      mbar_arrive(pfull);
    }
    if (warp == 1 || warp >= 2 + kSets * kSetWarps) {
      // ---------------------------------------------------------- MMA issuers
      // issuer i takes units n = i, i + kIssuers, ...: accumulator n % 2 = i and stages
      // of its own (kStages is even)
      const int iss = warp == 1 ? 0 : warp - (1 + kSets * kSetWarps);
      if (lane == 0 && mbar_wait(pfull, 0, kErrWaitFull)) {
        constexpr uint32_t idesc = idesc_bf16(kTok, kSlotCols);
        // Descriptors differ only in the start-address field (bits 0-13, address / 16).
        const uint64_t adesc0 = smem_desc(base, 16, 1024, 2);
        const uint64_t bdesc0 = smem_desc(pbase, 128, 512, 0);
        int stage = iss;
        uint32_t phase = 0;
        int pr = pr0 + iss;
        if (pr >= npair) pr -= npair;
        uint32_t n = static_cast<uint32_t>(iss);
        for (int64_t v = v_begin + iss; v < v_end; v += kIssuers, n += kIssuers) {
          const uint32_t a = n & 1u;
          if (!mbar_wait(full_bar(stage), phase, kErrWaitFull)) break;
          if (!mbar_wait(tempty(a), ((n >> 1) & 1u) ^ 1u, kErrWaitTmemEmpty)) break;
          tc_fence_after();
          const uint64_t ad = adesc0 + static_cast<uint32_t>(stage * (kStageBytes >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint32_t>(pr * (kPPairBytes >> 4));
          const uint32_t d = tmem_base + a * kAccCols;
#pragma unroll
          for (int j = 0; j < kBlk; ++j)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
              // A: block j is the j-th 64 bytes of the box's 128-byte rows, K-step 32 bytes;
              // B: block j's three terms (96 rows), K-step 256 bytes
              mma_bf16(d + j * kSlotCols, ad + ((j * 64 + ks * 32) >> 4),
                       bd + ((j * kPBlockBytes + ks * 256) >> 4), idesc, static_cast<uint32_t>(ks));
          tc_commit(tfull(a));
          tc_commit(empty_bar(stage));
          stage += kIssuers;
          if (stage >= kStages) { stage -= kStages; phase ^= 1u; }
          pr += kIssuers;
          while (pr >= npair) pr -= npair;
        }
        // every MMA issued above has finished before TMEM is released
        tc_commit(done_bar(iss));
        mbar_wait(done_bar(iss), 0, kErrWaitTmemFull);
      }
    } else {
      // ------------------------------------------------------ quantizer sets
      const int w = warp - 2;
      const int set = w / kSetWarps;       // units n with n % 2 == set
      const int j = (w >> 2) & 1;          // block of the pair
      const int q = warp & 3;              // TMEM lane quarter of this warp
      const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                              static_cast<uint32_t>(set) * kAccCols + j * kSlotCols;
      // unit state: token tile and pair index within the strip
      int64_t mt = mt0;
      int pr = pr0;
      if (set == 1 && ++pr == npair) { pr = 0; ++mt; }
      uint32_t k = 0;  // this set's units handled so far
      // the clip ratios were written by other warps: wait for all builders
      const bool ready = mbar_wait(pfull, 0, kErrWaitFull);
      for (int64_t v = v_begin + set; ready && v < v_end; v += kSets, ++k) {
        if (!mbar_wait(tfull(set), k & 1u, kErrWaitTmemFull)) break;
        tc_fence_after();
        // the three partial products y_hi, y_mid, y_lo, summed in that order
        uint32_t r[32], r2[32];
        tmem_ld_32x32b_x32(taddr0, r);
        tmem_ld_32x32b_x32(taddr0 + 32, r2);
        tmem_wait_ld();
        uint64_t y2[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          y2[c] = fadd2(pack2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])),
                        pack2(__uint_as_float(r2[2 * c]), __uint_as_float(r2[2 * c + 1])));
        tmem_ld_32x32b_x32(taddr0 + 64, r);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty(set));  // accumulator read: the issuer may reuse it
        float y[32];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          unpack2(fadd2(y2[c], pack2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1]))), y[2 * c],
                  y[2 * c + 1]);
        const int lb = 2 * pr + j;  // block within the strip
        const int64_t b = 2 * static_cast<int64_t>(pair_base) + lb;
        const int64_t m = mt * kTok + 32 * q + lane;  // token
        const bool valid = b < p.nb && m < p.rows;
        float r_lo, r_hi;
        if (kPerRowClip) {
          r_lo = (valid && p.g_lo) ? clip_ratio(p.g_lo[m * p.nb + b]) : 1.0f;
          r_hi = (valid && p.g_hi) ? clip_ratio(p.g_hi[m * p.nb + b]) : 1.0f;
        } else {
          r_lo = ratios[lb];
          r_hi = ratios[2 * kStrip + lb];
        }
        uint32_t packed[kFp8 ? 8 : 4];
        const uint32_t sbyte = quantize_block<kFp8>(y, r_lo, r_hi, packed);
        if constexpr (kKv) {
          if (valid) {
            const int64_t tok = m / p.kv_heads;
            const int64_t slot = p.slots[tok];
            if (slot >= p.kv_slots) {
              atomicOr(&g_dev_error, kErrBadIndex);
            } else if (slot >= 0) {
              const int64_t crow = slot * p.kv_heads + (m - tok * p.kv_heads);
              if constexpr (kFp8) {
                uint4* dst = reinterpret_cast<uint4*>(p.codes + crow * p.K + b * kG);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              } else {
                *reinterpret_cast<uint4*>(p.codes + crow * (p.K / 2) + b * (kG / 2)) =
                    make_uint4(packed[0], packed[1], packed[2], packed[3]);
              }
              p.scales[crow * p.nb + b] = static_cast<uint8_t>(sbyte);
            }
            if (kTrace) {
              float4* dst = reinterpret_cast<float4*>(p.y_out + m * p.K + b * kG);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
            }
          }
        } else {
          if (valid) {
            if constexpr (kFp8) {
              uint4* dst = reinterpret_cast<uint4*>(p.codes + m * p.K + b * kG);
              dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            } else {
              *reinterpret_cast<uint4*>(p.codes + m * (p.K / 2) + b * (kG / 2)) =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
            if (kTrace) {
              float4* dst = reinterpret_cast<float4*>(p.y_out + m * p.K + b * kG);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
            }
          }
          // rows past M and blocks past nb are padding of the tiled scale buffer: 0;
          // the last pair also covers the padding blocks [2*nbp2, 4*nbp4)
          uint8_t* sp = p.scales + scale_offset(m, b, p.nbp4);
          *sp = static_cast<uint8_t>(valid ? sbyte : 0u);
          if ((b & 3) < 2 && b + 2 >= 2 * static_cast<int64_t>(p.nbp2) && b + 2 < 4 * static_cast<int64_t>(p.nbp4))
            sp[2] = 0;
        }
        // next unit of this set
        pr += kSets;
        while (pr >= npair) { pr -= npair; ++mt; }
      }
    }
  }

  // with completion flags, the codes and scales are read by a running GEMM's tensor copies
  // (async proxy): every thread orders its stores before them here
  if (p.cta_flags != nullptr) asm volatile("fence.proxy.async.global;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
  // every thread's stores are done (barrier above): publish them for a GEMM that starts on
  // this CTA's token tiles. (Publishing every unit as it was stored instead, with one
  // GPU-scope release per unit from a warp of its own, made the prefill_o step 25 us
  // slower.)
  if (threadIdx.x == 0 && p.cta_flags != nullptr) {
    __threadfence();
    st_release_gpu_u64(p.cta_flags + blockIdx.x, p.epoch);
  }
}

__global__ void bat_clip_ratio_kernel(const float* g, int64_t n, float* r) {
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    r[t] = g ? clip_ratio(g[t]) : 1.0f;
}

}  // namespace bat
