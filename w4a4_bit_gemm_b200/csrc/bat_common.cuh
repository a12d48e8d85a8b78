// Device-side helpers shared by the BATQuant kernels: bf16 unpacking, packed
// fp32x2 FMA, E2M1 conversion, mbarrier / TMA / tcgen05 wrappers (inline PTX
// for sm_100a), and bounded waits that report a stall instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bat {

constexpr int kG = 32;  // MXFP4 block: elements per UE8M0 scale

// Sticky error word: kernels OR a code in when a bounded wait runs out.
__device__ unsigned int g_dev_error;

enum DevError : unsigned int {
  kErrWaitFull = 1u,
  kErrWaitEmpty = 2u,
  kErrWaitTmemFull = 4u,
  kErrWaitTmemEmpty = 8u,
  kErrBadIndex = 16u,  // a cache slot index outside [0, num_slots) (the access is skipped)
};

// fp32(sigma(g)) evaluated in fp64; +inf gives exactly 1.
__device__ __forceinline__ float clip_ratio(float g) {
  if (isinf(g) && g > 0.0f) return 1.0f;
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(g))));
}

__device__ __forceinline__ int64_t scale_offset(int64_t m, int64_t b, int nbp4) {
  return ((m >> 7) * nbp4 + (b >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (b & 3);
}

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// d = a * b + c on two fp32 lanes at once (sm_100 packed FMA), round-to-nearest.
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Two fp32 values -> one byte of E2M1 codes: `lo` in bits 0-3, `hi` in bits 4-7.
// Round-to-nearest-even with saturation to +-6 (the conversion instruction's
// .rn.satfinite behaviour; checked element by element against the oracle).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Eight fp32 values -> one word of E2M1 codes, v[i] in bits 4i..4i+3 (same rounding).
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// Four fp32 values -> one word of OCP E4M3 codes, v[i] in byte i (round to nearest
// even, saturating at +-448).
__device__ __forceinline__ uint32_t e4m3x4(float v0, float v1, float v2, float v3) {
  uint32_t r;
  asm("{\n\t.reg .b16 h0, h1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
      "mov.b32 %0, {h0, h1};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
  return r;
}

// 64-bit flag store with release / load with acquire, at GPU scope.
__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Shared-memory counter: add with release / load with acquire, at CTA scope.
__device__ __forceinline__ void red_release_cta_add(uint32_t addr, uint32_t v) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cta_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Warpgroup register reallocation (all four warps of a warpgroup execute it).
template <uint32_t kRegs>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start while the kernel before it on the stream is still
// running; grid_dependency_wait() returns once that kernel has completed and its
// memory operations are visible, so everything before it must not touch global
// memory other kernels write. allow_dependents() lets the next such kernel start.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_try_wait, but a thread whose phase is not complete yet may sleep in the
// instruction for up to `hint_ns` nanoseconds (it wakes when the phase completes),
// instead of spinning and taking issue slots from the warps that do the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of `bar` to complete, giving up after `limit_ns`
// nanoseconds: then the error word gets `code` and the caller unwinds.
constexpr uint64_t kWaitLimitNs = 4000000000ull;
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_dev_error, code);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA / bulk copies
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
// The same copy with an L2 cache-policy hint (e.g. evict-first for data read once).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
// L2 policy for a stream read once: its lines are the first to be evicted, so the stream
// does not push out data that is still wanted (measured: about 13 % more read bandwidth
// for a 134 MB stream of tensor copies).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Make this thread's generic-proxy shared-memory stores visible to the async proxy
// (TMA, tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
// Block-scaled MXFP4 MMA: D[tmem] (+)= (A * 2^sfa) x (B * 2^sfb)^T, M=128, K=64.
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// D (+)= A . B^T with one UE8M0 scale per 32 elements along K (K = 32 per
// instruction); A and B element types come from the instruction descriptor.
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Copy 32 rows x 16 bytes from shared memory into TMEM, replicated into all four
// 32-lane sub-partitions (the scale-factor layout the block-scaled MMA reads).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
// Thread t of the warp writes its registers to TMEM lane (lane base + t), consecutive columns.
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 columns of 32-bit words: thread t of the warp gets row (lane base + t).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format, version 1).
//   start, lbo, sbo in bytes; layout: 0 = no swizzle, 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((start >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of kind::mxf4 with UE8M0 scales, K-major A and B,
// fp32 accumulation. sf ids select which byte pair of the 32-bit TMEM scale word
// this MMA (K = 64, two scales per row) uses.
__host__ __device__ constexpr uint32_t idesc_mxf4(int m, int n, uint32_t a_sf_id,
                                                  uint32_t b_sf_id) {
  return (b_sf_id & 3u) << 4 |            // B scale-factor id
         1u << 7 |                        // A format: E2M1
         1u << 10 |                       // B format: E2M1
         static_cast<uint32_t>(n >> 3) << 17 |  // N / 8
         1u << 23 |                       // scale format UE8M0
         static_cast<uint32_t>(m >> 4) << 24 |  // M / 16
         (a_sf_id & 3u) << 29;            // A scale-factor id
}

// ---------------------------------------------------------------- row quantizer math
// kLs >= 0: the split as a constant; -1: read it from `ls_rt`. kGlobal: a and b point to
// global memory (read through the read-only cache); otherwise to shared memory.
template <int kLs, bool kGlobal = true>
__device__ __forceinline__ void rows_build_pc(float (&pc)[32][4], const float* __restrict__ a,
                                              const float* __restrict__ b, int bq, int u, int ls_rt) {
  const int ls = kLs >= 0 ? kLs : ls_rt;
  const int sm = (1 << ls) - 1, tt = 32 >> ls;
  const float* bb = b + static_cast<int64_t>(bq) * tt * tt;
#pragma unroll
  for (int k = 0; k < 32; ++k)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = 4 * u + j;
      const float* pb = bb + (k >> ls) * tt + (n >> ls);
      const float* pa = a + ((k & sm) << ls) + (n & sm);
      pc[k][j] = kGlobal ? __fmul_rn(__ldg(pb), __ldg(pa)) : __fmul_rn(*pb, *pa);
    }
}

// The 32 bf16 inputs of one block (64 bytes, 16-byte aligned) as fp32.
__device__ __forceinline__ void rows_load_block(const uint16_t* src16, float (&x)[32]) {
  const uint4* src = reinterpret_cast<const uint4*>(src16);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = src[c];
    x[8 * c + 0] = bf16lo(w.x); x[8 * c + 1] = bf16hi(w.x);
    x[8 * c + 2] = bf16lo(w.y); x[8 * c + 3] = bf16hi(w.y);
    x[8 * c + 4] = bf16lo(w.z); x[8 * c + 5] = bf16hi(w.z);
    x[8 * c + 6] = bf16lo(w.w); x[8 * c + 7] = bf16hi(w.w);
  }
}

// One block of one row, spread over the eight lanes (l & ~7) .. (l | 7) of the warp:
// this lane's transformed values y[j] = sum_k x[k] P_b[k][4u + j] (fp32, k ascending),
// the block clip and the MX scale (min / max over the eight lanes by shuffles, so the
// whole warp must call it together), and this lane's four codes: E2M1 in the low 16
// bits (element 4u in the lowest nibble) or E4M3 in 32 bits (4u in the lowest byte).
template <bool kFp8>
__device__ __forceinline__ void rows_block_quant(const float (&x)[32], const float (&pc)[32][4],
                                                 float r_lo, float r_hi, float (&y)[4],
                                                 uint32_t& code, int& sbyte) {
  uint64_t y01 = 0ull, y23 = 0ull;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint64_t xx = pack2(x[k], x[k]);
    y01 = ffma2(xx, pack2(pc[k][0], pc[k][1]), y01);
    y23 = ffma2(xx, pack2(pc[k][2], pc[k][3]), y23);
  }
  unpack2(y01, y[0], y[1]);
  unpack2(y23, y[2], y[3]);
  float mn = fminf(fminf(y[0], y[1]), fminf(y[2], y[3]));
  float mx = fmaxf(fmaxf(y[0], y[1]), fmaxf(y[2], y[3]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float lo = __fmul_rn(r_lo, mn);
  const float hi = __fmul_rn(r_hi, mx);
  const float amax = fmaxf(fabsf(fminf(fmaxf(mn, lo), hi)), fabsf(fminf(fmaxf(mx, lo), hi)));
  constexpr int kEmax = kFp8 ? 8 : 2;
  const int efield = static_cast<int>(__float_as_uint(amax) >> 23);
  sbyte = efield > kEmax ? efield - kEmax : 0;  // e + 127
  const float inv_scale = __uint_as_float(static_cast<uint32_t>(254 - sbyte) << 23);  // 2^-e
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __fmaf_rn(fminf(fmaxf(y[i], lo), hi), inv_scale, 0.0f);
  code = kFp8 ? e4m3x4(v[0], v[1], v[2], v[3]) : (e2m1x2(v[0], v[1]) | (e2m1x2(v[2], v[3]) << 8));
}

// Instruction descriptor of kind::mxf8f6f4 with A in E4M3 and B in E2M1 (format codes
// 0 and 5 of that kind), fp32 accumulation, UE8M0 scales, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_mxf8f6f4_e4m3_e2m1(int m, int n, uint32_t a_sf_id,
                                                                uint32_t b_sf_id) {
  return (b_sf_id & 3u) << 4 |            // B scale-factor id
         0u << 7 |                        // A format: E4M3
         5u << 10 |                       // B format: E2M1
         static_cast<uint32_t>(n >> 3) << 17 |  // N / 8
         1u << 23 |                       // scale format UE8M0
         static_cast<uint32_t>(m >> 4) << 24 |  // M / 16
         (a_sf_id & 3u) << 29;            // A scale-factor id
}

}  // namespace bat
