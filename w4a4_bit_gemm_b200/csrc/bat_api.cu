// C-ABI of the BATQuant W4A4 linear layer: host validation, launch
// configuration, tensor maps and the offline fp64 inverse of the weight side.
// Every kernel of the library is compiled in this one translation unit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/bat.h"
#include "bat_common.cuh"
#include "bat_gemm.cuh"
#include "bat_gemm2.cuh"
#include "bat_gemm_dec.cuh"
#include "bat_kv.cuh"
#include "bat_prologue.cuh"

namespace {

constexpr int64_t kMaxK = 262144;
// Rows of any operand (activations, weights, KV rows and cache slots x heads): the
// tensor-memory copies address a tile by 32-bit signed coordinates, so every tile
// origin must stay well below 2^31.
constexpr int64_t kMaxRows = int64_t(1) << 30;
constexpr double kMaxCond = 1e6;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// ---------------------------------------------------------------- device facts (cached)
struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 sm_100, 2 unsupported
  std::atomic<int> sms{0};
  std::atomic<int> gemm_attr{0};    // bit 0: W4A4 GEMM, bit 1: W4A8 GEMM attribute set
  std::atomic<int> pro_attr{0};     // bit t: the prologue variant t has its smem attribute set
  std::atomic<int> max_clusters[2][9];  // [W4A8][cluster size]: clusters resident at once, 0 unknown
  std::atomic<int> pair_attr{0};        // the CTA-pair GEMM's smem attribute is set
  std::atomic<int> max_pairs{0};        // CTA pairs of that GEMM resident at once, 0 unknown
  std::atomic<int> dec_attr{0};         // the decode GEMM's smem attribute is set
  std::atomic<int> dec_clusters[9];     // [cluster size]: its clusters resident at once, 0 unknown
};
DeviceInfo g_dev[64];

bat_status_t current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BAT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return BAT_ERR_UNSUPPORTED;
  DeviceInfo& d = g_dev[dev];
  int st = d.state.load();
  if (st == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BAT_ERR_CUDA;
    d.sms.store(sms);
    st = (major == 10 && minor == 0) ? 1 : 2;
    d.state.store(st);
  }
  if (st != 1) return BAT_ERR_UNSUPPORTED;
  *dev_out = dev;
  *sms_out = d.sms.load();
  return BAT_OK;
}

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

bat_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BAT_OK;
  t_last_cuda_error = e;
  return BAT_ERR_CUDA;
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load();
  if (f) return f;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  f = reinterpret_cast<EncodeTiledFn>(ptr);
  fn.store(f);
  return f;
}

// Codes of an MXFP4 matrix seen as a [rows][k/2] byte tensor, box of 128 bytes x box_rows,
// 128-byte swizzle (the K-major operand layout of the MMA).
bool make_code_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t k, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// E4M3 codes of an MXFP8 matrix, [rows][k] bytes, box of 128 bytes x box_rows, 128-byte
// swizzle.
bool make_code8_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t k, uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed E2M1 codes of an MXFP4 matrix as 4-bit elements [rows][k], loaded with the
// unpacking data type: every 16 elements (8 bytes in memory) land in 16 bytes of shared
// memory, the operand layout of kind::mxf8f6f4 for E2M1. Box of 128 elements (128 bytes
// in shared memory) x box_rows, 128-byte swizzle. Needs k % 128 == 0 and 32-byte
// aligned codes.
bool make_code4_unpack_map(CUtensorMap* map, const void* codes, int64_t rows, int64_t k,
                           uint32_t box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(codes), dims,
                 strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 Y [M][N] for the GEMM's TMA store: box of 64 columns (128 bytes) x 128 rows,
// 128-byte swizzle, matching the epilogue's staging layout. Needs N % 8 == 0.
bool make_out_map(CUtensorMap* map, void* y, int64_t M, int64_t N) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(bat::gemm::kBM)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 Y [M][N] for the CTA-pair GEMM's TMA store: box of 32 columns (64 bytes) x 128 rows,
// 64-byte swizzle, matching that epilogue's staging layout. Needs N % 8 == 0.
bool make_out_map64(CUtensorMap* map, void* y, int64_t M, int64_t N) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * 2)};
  cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(bat::gemm2::kRows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 X [rows][K] for the prologue: box of 64 columns (128 bytes) x 128 rows, 128-byte
// swizzle (the K-major A-operand layout of the transform MMA); rows past the end read 0.
bool make_act_map(CUtensorMap* map, const void* x, int64_t rows, int64_t K) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(bat::pro::kTok)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                 estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- fp64 inverse (host)
// Gauss-Jordan elimination with partial pivoting on an n x n row-major matrix.
// Returns false if a pivot vanishes or the 1-norm condition number exceeds kMaxCond.
bool invert(int n, const double* a_in, double* inv) {
  std::vector<double> a(a_in, a_in + n * n);
  for (int i = 0; i < n * n; ++i) inv[i] = 0.0;
  for (int i = 0; i < n; ++i) inv[i * n + i] = 1.0;
  double norm_a = 0.0;
  for (int c = 0; c < n; ++c) {
    double s = 0.0;
    for (int r = 0; r < n; ++r) s += std::fabs(a_in[r * n + c]);
    norm_a = std::fmax(norm_a, s);
  }
  for (int c = 0; c < n; ++c) {
    int piv = c;
    for (int r = c + 1; r < n; ++r)
      if (std::fabs(a[r * n + c]) > std::fabs(a[piv * n + c])) piv = r;
    const double pv = a[piv * n + c];
    if (!(std::fabs(pv) > 0.0) || !std::isfinite(pv)) return false;
    if (piv != c)
      for (int j = 0; j < n; ++j) {
        std::swap(a[c * n + j], a[piv * n + j]);
        std::swap(inv[c * n + j], inv[piv * n + j]);
      }
    for (int j = 0; j < n; ++j) {
      a[c * n + j] /= pv;
      inv[c * n + j] /= pv;
    }
    for (int r = 0; r < n; ++r) {
      if (r == c) continue;
      const double f = a[r * n + c];
      if (f == 0.0) continue;
      for (int j = 0; j < n; ++j) {
        a[r * n + j] -= f * a[c * n + j];
        inv[r * n + j] -= f * inv[c * n + j];
      }
    }
  }
  double norm_inv = 0.0;
  for (int c = 0; c < n; ++c) {
    double s = 0.0;
    for (int r = 0; r < n; ++r) s += std::fabs(inv[r * n + c]);
    norm_inv = std::fmax(norm_inv, s);
  }
  const double cond = norm_a * norm_inv;
  return std::isfinite(cond) && cond <= kMaxCond;
}

// ---------------------------------------------------------------- prologue launch
bat_status_t check_mxfp4(const bat_mxfp4_t* q, int64_t rows, int64_t k) {
  if (!q || !q->codes || !q->scales) return BAT_ERR_INVALID_ARG;
  if (q->rows != rows || q->k != k) return BAT_ERR_SHAPE;
  if (!aligned16(q->codes) || !aligned16(q->scales)) return BAT_ERR_ALIGN;
  return BAT_OK;
}

bat_status_t check_act_args(const void* X, int64_t M, int64_t K, const float* A, const float* B,
                            const float* g_lo, const float* g_hi, const bat_mxfp4_t* Xq) {
  if (!X || !A || !B || !Xq) return BAT_ERR_INVALID_ARG;
  if ((g_lo == nullptr) != (g_hi == nullptr)) return BAT_ERR_INVALID_ARG;
  if (M < 1 || K < 32) return BAT_ERR_INVALID_ARG;
  if (K % 32 != 0 || K > kMaxK || M > kMaxRows) return BAT_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B)) return BAT_ERR_ALIGN;
  return check_mxfp4(Xq, M, K);
}

// The CUDA-core row quantizer: activation rows (slots == null: codes [rows][D(/2)], tiled
// scales) or KV-cache rows (token row / H stored at cache slot slots[token]).
// Activation batches of at most this many rows run on the CUDA-core row quantizer
// (its latency is a few microseconds; the tensor-core prologue's set-up costs more).
constexpr int64_t kRowsCudaCore = 64;
// The linear layer's per-CTA completion flags (64-bit): the row quantizer's (at most 16
// warps per SM, two CTAs per SM) or the prologue's (one CTA per SM at most), and their
// epochs, unique per call and process (a salted counter), so flags left by earlier calls
// never match.
constexpr size_t kDoneFlagBytes = 4096;
std::atomic<unsigned long long> g_calls{0};
unsigned long long next_epoch() {
  static const unsigned long long salt =
      (static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count()) *
       0x9E3779B97F4A7C15ull) ^ static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(&g_calls));
  return (salt + 2 * g_calls.fetch_add(1)) | 1ull;  // odd, so never the 0 of fresh memory
}

// done_flags (activation rows only): one 64-bit completion flag per CTA, set to `epoch`;
// *grid_out gets the number of CTAs.
bat_status_t launch_rows(const void* x, int64_t rows, int64_t H, int64_t S,
                                const int64_t* slots, int64_t D, const float* A, const float* B,
                                const float* g_lo, const float* g_hi, int ls, bool fp8,
                                uint8_t* codes, uint8_t* scales, float* y_out, int sms,
                                cudaStream_t s, unsigned long long* done_flags = nullptr,
                                unsigned long long epoch = 0, int* grid_out = nullptr) {
  bat::RowQuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.a = A;
  p.b = B;
  p.g_lo = g_lo;
  p.g_hi = g_hi;
  p.codes = codes;
  p.scales = scales;
  p.y_out = y_out;
  p.slots = slots;
  p.rows = rows;
  p.H = H;
  p.S = S;
  p.D = static_cast<int>(D);
  p.nb = static_cast<int>(D / 32);
  p.groups = (p.nb + 3) / 4;
  p.ls = ls;
  p.nbp4 = (p.nb + 3) / 4;
  p.done_flags = slots == nullptr ? done_flags : nullptr;
  p.epoch = epoch;
  if (grid_out) *grid_out = 0;
  // about 16 warps per SM in all, each group of blocks over a stride of R rows
  int64_t R = static_cast<int64_t>(sms) * 16 / p.groups;
  if (R > rows) R = rows;
  if (R < 1) R = 1;
  p.R = static_cast<int>(R);
  const int64_t warps = static_cast<int64_t>(p.groups) * R;
  const unsigned grid = static_cast<unsigned>((warps + bat::kv::kWarps - 1) / bat::kv::kWarps);
  if (grid > kDoneFlagBytes / 8) p.done_flags = nullptr;  // (never at supported sizes)
  if (grid_out) *grid_out = p.done_flags != nullptr ? static_cast<int>(grid) : 0;
  const bool kv = slots != nullptr, tr = y_out != nullptr;
  void (*k)(bat::RowQuantParams);
  if (kv)
    k = fp8 ? (tr ? bat::bat_rows_quantize_kernel<true, true, true> : bat::bat_rows_quantize_kernel<true, false, true>)
            : (tr ? bat::bat_rows_quantize_kernel<false, true, true> : bat::bat_rows_quantize_kernel<false, false, true>);
  else
    k = fp8 ? (tr ? bat::bat_rows_quantize_kernel<true, true, false> : bat::bat_rows_quantize_kernel<true, false, false>)
            : (tr ? bat::bat_rows_quantize_kernel<false, true, false> : bat::bat_rows_quantize_kernel<false, false, false>);
  k<<<grid, bat::kv::kThreads, 0, s>>>(p);
  return cuda_status(cudaGetLastError());
}

bat_status_t launch_prologue(const void* X, int64_t rows, int64_t K, const float* A,
                             const float* B, const float* g_lo, const float* g_hi, bool per_row,
                             const bat_mxfp4_t* out, float* y_out, cudaStream_t stream,
                             int ls = 3, bool fp8 = false, const int64_t* kv_slots = nullptr,
                             int64_t kv_heads = 0, int64_t kv_nslots = 0,
                             unsigned long long* done_flags = nullptr, unsigned long long epoch = 0,
                             int* rows_grid_out = nullptr, unsigned long long* cta_flags = nullptr,
                             int* strips_out = nullptr, int* cps_out = nullptr) {
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  if (rows >= (int64_t{1} << 31)) return BAT_ERR_SHAPE;  // TMA row coordinates are int32
  if (!per_row && kv_slots == nullptr && rows <= kRowsCudaCore)
    return launch_rows(X, rows, 1, 0, nullptr, K, A, B, g_lo, g_hi, ls, fp8,
                       static_cast<uint8_t*>(out->codes), static_cast<uint8_t*>(out->scales), y_out,
                       sms, stream, done_flags, epoch, rows_grid_out);
  CUtensorMap tx;
  if (!make_act_map(&tx, X, rows, K)) return BAT_ERR_CUDA;
  bat::PrologueParams p;
  p.a = A;
  p.b = B;
  p.g_lo = g_lo;
  p.g_hi = g_hi;
  p.codes = static_cast<uint8_t*>(out->codes);
  p.scales = static_cast<uint8_t*>(out->scales);
  p.y_out = y_out;
  p.rows = rows;
  p.K = K;
  p.nb = static_cast<int>(K / 32);
  p.ls = ls;
  p.slots = kv_slots;
  // unit completion flags: activations of the linear layer only
  p.cta_flags = (!per_row && kv_slots == nullptr && !fp8) ? cta_flags : nullptr;
  p.epoch = epoch;
  p.kv_heads = kv_heads;
  p.kv_slots = kv_nslots;
  p.nbp2 = (p.nb + 1) / 2;
  p.nbp4 = (p.nb + 3) / 4;
  p.mtiles = (rows + bat::pro::kTok - 1) / bat::pro::kTok;
  p.strips = (p.nbp2 + bat::pro::kStrip - 1) / bat::pro::kStrip;
  // CTAs per strip: the SMs shared out over the strips, but no more CTAs than a
  // strip has units
  {
    int cps = sms / p.strips;
    const int64_t strip_units = p.mtiles * (p.nbp2 < bat::pro::kStrip ? p.nbp2 : bat::pro::kStrip);
    if (cps > strip_units) cps = static_cast<int>(strip_units);
    p.cps = cps < 1 ? 1 : cps;
  }
  void (*kern)(CUtensorMap, bat::PrologueParams);
  const bool kv = kv_slots != nullptr;
  if (kv) {  // KV-cache store: rows are (token, head), codes and scales go to cache slots
    if (fp8)
      kern = y_out ? bat::bat_prologue_kernel<true, false, true, true>
                   : bat::bat_prologue_kernel<false, false, true, true>;
    else
      kern = y_out ? bat::bat_prologue_kernel<true, false, false, true>
                   : bat::bat_prologue_kernel<false, false, false, true>;
  } else if (fp8)  // activations only: clip logits per block
    kern = y_out ? bat::bat_prologue_kernel<true, false, true> : bat::bat_prologue_kernel<false, false, true>;
  else if (per_row)
    kern = y_out ? bat::bat_prologue_kernel<true, true> : bat::bat_prologue_kernel<false, true>;
  else
    kern = y_out ? bat::bat_prologue_kernel<true, false> : bat::bat_prologue_kernel<false, false>;
  DeviceInfo& d = g_dev[dev];
  const int variant_bit =
      1 << ((kv ? 6 + (fp8 ? 2 : 0) : (fp8 ? 4 : (per_row ? 2 : 0))) + (y_out ? 1 : 0));
  if (!(d.pro_attr.load() & variant_bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bat::pro::kSmemBytes) != cudaSuccess)
      return BAT_ERR_CUDA;
    d.pro_attr.fetch_or(variant_bit);
  }
  // One CTA per (strip, part): about one per SM.
  const int64_t grid = static_cast<int64_t>(p.strips) * p.cps;
  if (strips_out) *strips_out = p.strips;
  if (cps_out) *cps_out = p.cps;
  kern<<<static_cast<unsigned>(grid), bat::pro::kThreads, bat::pro::kSmemBytes, stream>>>(tx, p);
  return cuda_status(cudaGetLastError());
}

// a8: Xq holds MXFP8 (E4M3) activations and the W4A8 kernel runs; K % 128 == 0 then.
// w_static: the kernel before the GEMM on the stream does not write the weights (the
// linear layer: that kernel is the activation quantizer). q_flags / q_ctas / epoch: that
// quantizer's completion flags (row quantizer), which the decode GEMM waits on instead of
// the grid dependency; null otherwise.
// cta_flags (CTA-pair kernel): the prologue's per-CTA completion flags (q_strips x q_cps
// CTAs), waited for tile by tile instead of the grid dependency (the tile-level overlap
// of the fused linear layer).
bat_status_t launch_gemm(const bat_mxfp4_t* Xq, const bat_mxfp4_t* Wq, void* Y,
                         bat_out_dtype_t out_dtype, cudaStream_t stream, bool a8 = false,
                         bool w_static = false, const unsigned long long* q_flags = nullptr,
                         int q_ctas = 0, unsigned long long epoch = 0,
                         const unsigned long long* cta_flags = nullptr, int q_strips = 0,
                         int q_cps = 0) {
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  CUtensorMap ta, tb, ty;
  if (a8) {
    if (!make_code8_map(&ta, Xq->codes, Xq->rows, Xq->k, bat::gemm::kBM)) return BAT_ERR_CUDA;
    if (!make_code4_unpack_map(&tb, Wq->codes, Wq->rows, Wq->k, bat::gemm::kBN)) return BAT_ERR_CUDA;
  } else {
    if (!make_code_map(&ta, Xq->codes, Xq->rows, Xq->k, bat::gemm::kBM)) return BAT_ERR_CUDA;
    if (!make_code_map(&tb, Wq->codes, Wq->rows, Wq->k, bat::gemm::kBN)) return BAT_ERR_CUDA;
  }
  std::memset(&ty, 0, sizeof(ty));
  bat::GemmParams p{};
  p.sfa = static_cast<const uint8_t*>(Xq->scales);
  p.sfb = static_cast<const uint8_t*>(Wq->scales);
  p.y = Y;
  p.M = Xq->rows;
  p.N = Wq->rows;
  p.K = Xq->k;
  p.nbp4 = static_cast<int>((Xq->k / 32 + 3) / 4);
  p.out_f32 = out_dtype == BAT_OUT_F32 ? 1 : 0;
  p.vec_ok = (p.N % (p.out_f32 ? 4 : 8)) == 0 ? 1 : 0;
  // bf16 output with 16-byte rows goes through shared-memory staging and TMA stores
  p.tma_store = (!p.out_f32 && p.vec_ok) ? 1 : 0;
  if (p.tma_store && !make_out_map(&ty, Y, p.M, p.N)) return BAT_ERR_CUDA;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, bat::GemmParams) =
      a8 ? bat::bat_mxf4_gemm_kernel<true> : bat::bat_mxf4_gemm_kernel<false>;
  const int smem = a8 ? bat::gemm::Cfg<true>::kSmemBytes : bat::gemm::Cfg<false>::kSmemBytes;
  const int64_t m_tiles = (p.M + bat::gemm::kBM - 1) / bat::gemm::kBM;
  const int64_t tiles = m_tiles * ((p.N + bat::gemm::kBN - 1) / bat::gemm::kBN);
  // Split-K over a cluster per tile when one row of tiles leaves most SMs idle (decode
  // shapes): up to 8 CTAs per tile, at least one K stage each.
  const int64_t k_stages = (p.K + (a8 ? 127 : 255)) / (a8 ? 128 : 256);
  DeviceInfo& d = g_dev[dev];
  const int64_t dks = (p.K + bat::gemmd::kBK - 1) / bat::gemmd::kBK;
  if (!a8 && p.M <= bat::gemmd::kMaxNx && dks <= bat::gemmd::kStages * bat::gemmd::kMaxSplits) {
    // decode shapes: Y^T = Wq . Xq^T on 128-row W tiles, K split over a cluster of S CTAs
    // per tile (bat_gemm_dec.cuh): the smallest power of two S that leaves each CTA at most
    // kStages K stages, doubled while the doubled grid still fits the SMs in one wave
    const int nx = static_cast<int>((p.M + 15) / 16 * 16);
    CUtensorMap tw;
    if (!make_code_map(&tw, Wq->codes, Wq->rows, Wq->k, bat::gemmd::kBM)) return BAT_ERR_CUDA;
    if (q_ctas <= 0) q_flags = nullptr;
    void (*dk)(CUtensorMap, bat::GemmParams, const uint8_t*, int, int, const unsigned long long*, int,
               unsigned long long) = bat::bat_mxf4_gemm_dec_kernel;
    if (!d.dec_attr.load()) {
      const cudaError_t ae = cudaFuncSetAttribute(dk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  bat::gemmd::kSmemBytes);
      if (ae != cudaSuccess) return cuda_status(ae);
      d.dec_attr.store(1);
    }
    const int64_t wt = (p.N + bat::gemmd::kBM - 1) / bat::gemmd::kBM;
    int S = 1;
    while (S * bat::gemmd::kStages < dks) S *= 2;
    while (2 * S <= bat::gemmd::kMaxSplits && 2 * S <= dks && wt * 2 * S <= sms) S *= 2;
    if (S > 1) {
      int n = d.dec_clusters[S].load();
      if (n == 0) {
        cudaLaunchConfig_t oc = {};
        oc.gridDim = dim3(static_cast<unsigned>(wt * S));
        oc.blockDim = dim3(bat::gemmd::kThreads);
        oc.dynamicSmemBytes = bat::gemmd::kSmemBytes;
        cudaLaunchAttribute ca[1];
        ca[0].id = cudaLaunchAttributeClusterDimension;
        ca[0].val.clusterDim.x = static_cast<unsigned>(S);
        ca[0].val.clusterDim.y = 1;
        ca[0].val.clusterDim.z = 1;
        oc.attrs = ca;
        oc.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, dk, &oc) != cudaSuccess || n < 1) n = -1;
        d.dec_clusters[S].store(n);
      }
      if (n < 1) return BAT_ERR_UNSUPPORTED;  // clusters of S CTAs cannot be resident
    }
    p.splits = S;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(wt * S));
    cfg.blockDim = dim3(bat::gemmd::kThreads);
    cfg.dynamicSmemBytes = bat::gemmd::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(S);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = S > 1 ? 2 : 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, dk, tw, p, static_cast<const uint8_t*>(Xq->codes), nx,
                                          w_static ? 1 : 0, q_flags, q_ctas, epoch));
  }
  const int variant_bit = a8 ? 2 : 1;
  if (!(d.gemm_attr.load() & variant_bit)) {
    const cudaError_t ae =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (ae != cudaSuccess) return cuda_status(ae);
    d.gemm_attr.fetch_or(variant_bit);
  }
  int64_t splits = 1;
  if (m_tiles == 1 && 2 * tiles <= sms) {
    splits = sms / tiles;
    if (splits > 8) splits = 8;
    if (splits > k_stages) splits = k_stages;
    // the largest cluster size whose clusters all fit on the GPU at once (one wave)
    for (; splits > 1; --splits) {
      std::atomic<int>& mc = d.max_clusters[a8 ? 1 : 0][splits];
      int n = mc.load();
      if (n == 0) {
        cudaLaunchConfig_t oc = {};
        oc.gridDim = dim3(static_cast<unsigned>(tiles * splits));
        oc.blockDim = dim3(bat::gemm::kThreads);
        oc.dynamicSmemBytes = smem;
        cudaLaunchAttribute ca[1];
        ca[0].id = cudaLaunchAttributeClusterDimension;
        ca[0].val.clusterDim.x = static_cast<unsigned>(splits);
        ca[0].val.clusterDim.y = 1;
        ca[0].val.clusterDim.z = 1;
        oc.attrs = ca;
        oc.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &oc) != cudaSuccess || n < 1) n = -1;
        mc.store(n);
      }
      if (n >= tiles) break;
    }
  }
  p.splits = static_cast<int>(splits);
  if (!a8 && splits == 1 && m_tiles >= 2) {
    // CTA pairs on 256 x 256 tiles (bat_gemm2.cuh)
    if (cta_flags != nullptr && q_strips > 0 && q_cps > 0) {
      static_assert(bat::pro::kStrip == 4, "the pair kernel's flag walk assumes 4 pairs per strip");
      p.cta_flags = cta_flags;
      p.q_mtiles = (p.M + 127) / 128;
      p.q_nbp2 = static_cast<int>((p.K / 32 + 1) / 2);
      p.q_strips = q_strips;
      p.q_cps = q_cps;
      p.q_epoch = epoch;
    }
    CUtensorMap pa, pb, py;
    if (!make_code_map(&pa, Xq->codes, Xq->rows, Xq->k, bat::gemm2::kRows)) return BAT_ERR_CUDA;
    if (!make_code_map(&pb, Wq->codes, Wq->rows, Wq->k, bat::gemm2::kBN / 2)) return BAT_ERR_CUDA;
    std::memset(&py, 0, sizeof(py));
    if (p.tma_store && !make_out_map64(&py, Y, p.M, p.N)) return BAT_ERR_CUDA;
    void (*pk)(CUtensorMap, CUtensorMap, CUtensorMap, bat::GemmParams) = bat::bat_mxf4_gemm_pair_kernel;
    if (!d.pair_attr.load()) {
      const cudaError_t ae = cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  bat::gemm2::kSmemBytes);
      if (ae != cudaSuccess) return cuda_status(ae);
      d.pair_attr.store(1);
    }
    const int64_t tiles2 = ((p.M + 255) / 256) * ((p.N + bat::gemm2::kBN - 1) / bat::gemm2::kBN);
    int npair = d.max_pairs.load();
    if (npair == 0) {
      cudaLaunchConfig_t oc = {};
      oc.gridDim = dim3(static_cast<unsigned>(sms & ~1));
      oc.blockDim = dim3(bat::gemm2::kThreads);
      oc.dynamicSmemBytes = bat::gemm2::kSmemBytes;
      cudaLaunchAttribute ca[1];
      ca[0].id = cudaLaunchAttributeClusterDimension;
      ca[0].val.clusterDim.x = 2;
      ca[0].val.clusterDim.y = 1;
      ca[0].val.clusterDim.z = 1;
      oc.attrs = ca;
      oc.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&npair, pk, &oc) != cudaSuccess || npair < 1) npair = sms / 2;
      d.max_pairs.store(npair);
    }
    const int64_t pairs = tiles2 < npair ? tiles2 : npair;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(bat::gemm2::kThreads);
    cfg.dynamicSmemBytes = bat::gemm2::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cuda_status(cudaLaunchKernelEx(&cfg, pk, pa, pb, py, p));
  }
  const int grid = splits > 1 ? static_cast<int>(tiles * splits)
                              : static_cast<int>(tiles < sms ? tiles : sms);
  // Programmatic stream serialization: the kernel's set-up may overlap the previous
  // kernel on the stream; it waits for that kernel's completion (griddepcontrol.wait)
  // before touching the operands or Y, so the stream order of results is unchanged.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(bat::gemm::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(splits);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = splits > 1 ? 2 : 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
}

bat_status_t check_gemm_args(const bat_mxfp4_t* Xq, const bat_mxfp4_t* Wq, const void* Y,
                             bat_out_dtype_t out_dtype, bool a8 = false) {
  if (!Xq || !Wq || !Y) return BAT_ERR_INVALID_ARG;
  if (out_dtype != BAT_OUT_BF16 && out_dtype != BAT_OUT_F32) return BAT_ERR_INVALID_ARG;
  if (Xq->rows < 1 || Wq->rows < 1 || Xq->k < 32) return BAT_ERR_INVALID_ARG;
  if (Xq->k != Wq->k || Xq->k % 32 != 0 || Xq->k > kMaxK) return BAT_ERR_SHAPE;
  if (Xq->rows > kMaxRows || Wq->rows > kMaxRows) return BAT_ERR_SHAPE;
  if (a8) {
    // the unpacking load of the weights: k % 128 == 0, 32-byte aligned codes
    if (Xq->k % 128 != 0) return BAT_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(Wq->codes) & 31u) != 0) return BAT_ERR_ALIGN;
  }
  bat_status_t st = check_mxfp4(Xq, Xq->rows, Xq->k);
  if (st != BAT_OK) return st;
  st = check_mxfp4(Wq, Wq->rows, Wq->k);
  if (st != BAT_OK) return st;
  if (!aligned16(Y)) return BAT_ERR_ALIGN;
  return BAT_OK;
}

}  // namespace

extern "C" {

int bat_version(void) { return 100; }

const char* bat_status_string(bat_status_t s) {
  switch (s) {
    case BAT_OK: return "BAT_OK";
    case BAT_ERR_INVALID_ARG: return "BAT_ERR_INVALID_ARG";
    case BAT_ERR_SHAPE: return "BAT_ERR_SHAPE";
    case BAT_ERR_ALIGN: return "BAT_ERR_ALIGN";
    case BAT_ERR_SINGULAR: return "BAT_ERR_SINGULAR";
    case BAT_ERR_CUDA: return "BAT_ERR_CUDA";
    case BAT_ERR_UNSUPPORTED: return "BAT_ERR_UNSUPPORTED";
    case BAT_ERR_WORKSPACE: return "BAT_ERR_WORKSPACE";
    case BAT_ERR_DEVICE: return "BAT_ERR_DEVICE";
  }
  return "BAT_ERR_UNKNOWN";
}

size_t bat_mxfp4_codes_bytes(int64_t rows, int64_t k) {
  if (rows < 1 || k < 32 || k % 32 != 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k / 2);
}

size_t bat_mxfp4_scales_bytes(int64_t rows, int64_t k) {
  if (rows < 1 || k < 32 || k % 32 != 0) return 0;
  const int64_t nbp4 = (k / 32 + 3) / 4;
  return static_cast<size_t>(round_up(rows, 128) / 128) * static_cast<size_t>(nbp4) * 512u;
}

bat_status_t bat_quantize_act(const void* X, int64_t M, int64_t K, const float* A, const float* B,
                              const float* g_lo, const float* g_hi, const bat_mxfp4_t* Xq,
                              void* stream) {
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, Xq);
  if (st != BAT_OK) return st;
  return launch_prologue(X, M, K, A, B, g_lo, g_hi, false, Xq, nullptr,
                         static_cast<cudaStream_t>(stream));
}

bat_status_t bat_quantize_act_trace(const void* X, int64_t M, int64_t K, const float* A,
                                    const float* B, const float* g_lo, const float* g_hi,
                                    const bat_mxfp4_t* Xq, float* y_out, void* stream) {
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, Xq);
  if (st != BAT_OK) return st;
  if (!y_out) return BAT_ERR_INVALID_ARG;
  if (!aligned16(y_out)) return BAT_ERR_ALIGN;
  return launch_prologue(X, M, K, A, B, g_lo, g_hi, false, Xq, y_out,
                         static_cast<cudaStream_t>(stream));
}

bat_status_t bat_clip_ratios(const float* g, int64_t n, float* r, void* stream) {
  if (!r || n < 1) return BAT_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  bat::bat_clip_ratio_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0,
                               static_cast<cudaStream_t>(stream)>>>(g, n, r);
  return cuda_status(cudaGetLastError());
}

bat_status_t bat_e2m1_encode(const float* v, int64_t n, uint8_t* codes, void* stream);

// log2 of a supported shared-factor size (1, 2, 4, ..., 32), or -1.
static int shared_log2(int shared) {
  for (int l = 0; l <= 5; ++l)
    if (shared == (1 << l)) return l;
  return -1;
}

bat_status_t bat_quantize_act_gpk(const void* X, int64_t M, int64_t K, const float* A, int shared,
                                  const float* B, const float* g_lo, const float* g_hi,
                                  const bat_mxfp4_t* Xq, float* y_out, void* stream) {
  const int ls = shared_log2(shared);
  if (ls < 0) return BAT_ERR_UNSUPPORTED;
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, Xq);
  if (st != BAT_OK) return st;
  if (y_out && !aligned16(y_out)) return BAT_ERR_ALIGN;
  return launch_prologue(X, M, K, A, B, g_lo, g_hi, false, Xq, y_out,
                         static_cast<cudaStream_t>(stream), ls);
}

bat_status_t bat_prepare_weight_gpk(const void* W, int64_t N, int64_t K, const float* A, int shared,
                                    const float* B, const float* gw_lo, const float* gw_hi,
                                    const bat_mxfp4_t* Wq, float* wt_out, void* stream) {
  const int ls = shared_log2(shared);
  if (ls < 0) return BAT_ERR_UNSUPPORTED;
  if (!W || !A || !B || !Wq) return BAT_ERR_INVALID_ARG;
  if ((gw_lo == nullptr) != (gw_hi == nullptr)) return BAT_ERR_INVALID_ARG;
  if (N < 1 || K < 32) return BAT_ERR_INVALID_ARG;
  if (K % 32 != 0 || K > kMaxK || N > kMaxRows) return BAT_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(A) || !aligned16(B)) return BAT_ERR_ALIGN;
  if (wt_out && !aligned16(wt_out)) return BAT_ERR_ALIGN;
  bat_status_t st = check_mxfp4(Wq, N, K);
  if (st != BAT_OK) return st;
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sa = shared, tb = 32 / shared;
  const int64_t nb = K / 32;
  std::vector<float> ha(static_cast<size_t>(sa) * sa), hb(static_cast<size_t>(nb) * tb * tb);
  if (cudaMemcpyAsync(ha.data(), A, ha.size() * sizeof(float), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(hb.data(), B, hb.size() * sizeof(float), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return BAT_ERR_CUDA;
  // Inverse-transposed factors: w_b (B_b^-T (x) A^-T) = vec_row(B_b^-1 W_r A^-T), which the
  // prologue computes as vec_row(F_b^T W_r G) with G = A^-T and F_b = B_b^-T. G is padded to
  // a multiple of four floats so that the F_b start 16-byte aligned.
  const size_t a_len = (static_cast<size_t>(sa) * sa + 3) & ~size_t{3};
  std::vector<float> fac(a_len + hb.size(), 0.0f);
  {
    std::vector<double> a(ha.begin(), ha.end()), inv(ha.size());
    if (!invert(sa, a.data(), inv.data())) return BAT_ERR_SINGULAR;
    for (int p = 0; p < sa; ++p)
      for (int q = 0; q < sa; ++q) fac[p * sa + q] = static_cast<float>(inv[q * sa + p]);
  }
  {
    std::vector<double> m(static_cast<size_t>(tb) * tb), inv(m.size());
    for (int64_t b = 0; b < nb; ++b) {
      const float* src = hb.data() + b * tb * tb;
      for (int i = 0; i < tb * tb; ++i) m[i] = src[i];
      if (!invert(tb, m.data(), inv.data())) return BAT_ERR_SINGULAR;
      float* dst = fac.data() + a_len + b * tb * tb;
      for (int i = 0; i < tb; ++i)
        for (int j = 0; j < tb; ++j) dst[i * tb + j] = static_cast<float>(inv[j * tb + i]);
    }
  }
  // Offline only: one temporary device buffer for the inverse factors (stream-ordered).
  void* dfac = nullptr;
  if (cudaMallocAsync(&dfac, fac.size() * sizeof(float), s) != cudaSuccess) return BAT_ERR_CUDA;
  st = cuda_status(cudaMemcpyAsync(dfac, fac.data(), fac.size() * sizeof(float),
                                   cudaMemcpyHostToDevice, s));
  if (st == BAT_OK) {
    const float* da = static_cast<const float*>(dfac);
    st = launch_prologue(W, N, K, da, da + a_len, gw_lo, gw_hi, true, Wq, wt_out, s, ls);
  }
  cudaFreeAsync(dfac, s);
  // `fac` is read by the async copy: wait before it goes out of scope.
  if (cudaStreamSynchronize(s) != cudaSuccess) return BAT_ERR_CUDA;
  return st;
}

bat_status_t bat_prepare_weight(const void* W, int64_t N, int64_t K, const float* A,
                                const float* B, const float* gw_lo, const float* gw_hi,
                                const bat_mxfp4_t* Wq, float* wt_out, void* stream) {
  return bat_prepare_weight_gpk(W, N, K, A, 8, B, gw_lo, gw_hi, Wq, wt_out, stream);
}

bat_status_t bat_block_hadamard_factors(int shared, int64_t nb, float* A, float* B) {
  const int ls = shared_log2(shared);
  if (ls < 0) return BAT_ERR_UNSUPPORTED;
  if (!A || !B || nb < 1) return BAT_ERR_INVALID_ARG;
  // Sylvester order: H_n[i][j] = (-1)^popcount(i & j), normalised by 1/sqrt(n).
  auto fill = [](int n, float* h) {
    const float c = static_cast<float>(1.0 / std::sqrt(static_cast<double>(n)));
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) h[i * n + j] = (__builtin_popcount(i & j) & 1) ? -c : c;
  };
  const int tb = 32 / shared;
  fill(shared, A);
  for (int64_t b = 0; b < nb; ++b) fill(tb, B + b * tb * tb);
  return BAT_OK;
}

bat_status_t bat_mxfp4_gemm(const bat_mxfp4_t* Xq, const bat_mxfp4_t* Wq, void* Y,
                            bat_out_dtype_t out_dtype, void* stream) {
  bat_status_t st = check_gemm_args(Xq, Wq, Y, out_dtype);
  if (st != BAT_OK) return st;
  return launch_gemm(Xq, Wq, Y, out_dtype, static_cast<cudaStream_t>(stream));
}

size_t bat_mxfp8_codes_bytes(int64_t rows, int64_t k) {
  if (rows < 1 || k < 32 || k % 32 != 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k);
}

bat_status_t bat_quantize_act_mxfp8(const void* X, int64_t M, int64_t K, const float* A,
                                    int shared, const float* B, const float* g_lo,
                                    const float* g_hi, const bat_mxfp8_t* Xq, float* y_out,
                                    void* stream) {
  const int ls = shared_log2(shared);
  if (ls < 0) return BAT_ERR_UNSUPPORTED;
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, Xq);
  if (st != BAT_OK) return st;
  if (y_out && !aligned16(y_out)) return BAT_ERR_ALIGN;
  return launch_prologue(X, M, K, A, B, g_lo, g_hi, false, Xq, y_out,
                         static_cast<cudaStream_t>(stream), ls, true);
}

size_t bat_kv_codes_bytes(int64_t num_slots, int64_t H, int64_t D, bat_kv_format_t fmt) {
  if (num_slots < 1 || H < 1 || D < 32 || D % 32 != 0) return 0;
  if (fmt != BAT_KV_MXFP8 && fmt != BAT_KV_MXFP4) return 0;
  const size_t n = static_cast<size_t>(num_slots) * static_cast<size_t>(H) * static_cast<size_t>(D);
  return fmt == BAT_KV_MXFP8 ? n : n / 2;
}

size_t bat_kv_scales_bytes(int64_t num_slots, int64_t H, int64_t D) {
  if (num_slots < 1 || H < 1 || D < 32 || D % 32 != 0) return 0;
  return static_cast<size_t>(num_slots) * static_cast<size_t>(H) * static_cast<size_t>(D / 32);
}

static bat_status_t kv_shape_check(int64_t T, int64_t H, int64_t D, int64_t num_slots, int shared,
                                   int* ls) {
  *ls = shared_log2(shared);
  if (*ls < 0) return BAT_ERR_UNSUPPORTED;
  if (T < 1 || H < 1 || num_slots < 1) return BAT_ERR_INVALID_ARG;
  if (D < 32 || D % 32 != 0 || D > 32 * bat::kv::kMaxBlocks) return BAT_ERR_SHAPE;
  // (token, head) rows and cache rows, without forming a product that could overflow
  if (H > kMaxRows || T > kMaxRows / H || num_slots > kMaxRows / H) return BAT_ERR_SHAPE;
  return BAT_OK;
}

// (token, head) rows from which bat_kv_quantize runs the tensor-core prologue
// instead of the CUDA-core kernel
constexpr int64_t kKvTensorRows = 4096;

static unsigned kv_grid(int64_t items, int sms) {
  const int64_t want = (items + bat::kv::kWarps - 1) / bat::kv::kWarps;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  return static_cast<unsigned>(want < cap ? want : cap);
}

bat_status_t bat_kv_quantize(const void* kv, int64_t T, int64_t H, int64_t D, const float* A,
                             int shared, const float* B, const float* g_lo, const float* g_hi,
                             const int64_t* slots, bat_kv_format_t fmt, void* cache_codes,
                             void* cache_scales, int64_t num_slots, float* y_out, void* stream) {
  int ls = 0;
  bat_status_t st = kv_shape_check(T, H, D, num_slots, shared, &ls);
  if (st != BAT_OK) return st;
  if (fmt != BAT_KV_MXFP8 && fmt != BAT_KV_MXFP4) return BAT_ERR_INVALID_ARG;
  if (!kv || !A || !B || !slots || !cache_codes || !cache_scales) return BAT_ERR_INVALID_ARG;
  if ((g_lo == nullptr) != (g_hi == nullptr)) return BAT_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(cache_codes) || !aligned16(A) || !aligned16(B) ||
      (reinterpret_cast<uintptr_t>(slots) & 7u) != 0 || (y_out && !aligned16(y_out)))
    return BAT_ERR_ALIGN;
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool fp8 = fmt == BAT_KV_MXFP8;
  if (T * H >= kKvTensorRows) {
    // a prefill-sized batch: the tensor-core prologue over the (token, head) rows
    if (T * H >= (int64_t{1} << 31)) return BAT_ERR_SHAPE;
    bat_mxfp4_t out;
    out.codes = cache_codes;
    out.scales = cache_scales;
    out.rows = T * H;
    out.k = D;
    return launch_prologue(kv, T * H, D, A, B, g_lo, g_hi, false, &out, y_out, s, ls, fp8, slots,
                           H, num_slots);
  }
  return launch_rows(kv, T * H, H, num_slots, slots, D, A, B, g_lo, g_hi, ls, fp8,
                     static_cast<uint8_t*>(cache_codes), static_cast<uint8_t*>(cache_scales), y_out,
                     sms, s);
}

bat_status_t bat_kv_dequantize(const void* cache_codes, const void* cache_scales,
                               int64_t num_slots, int64_t H, int64_t D, bat_kv_format_t fmt,
                               const int64_t* slots, int64_t T, const float* A, int shared,
                               const float* B, void* out, bat_out_dtype_t out_dtype,
                               void* stream) {
  int ls = 0;
  bat_status_t st = kv_shape_check(T, H, D, num_slots, shared, &ls);
  if (st != BAT_OK) return st;
  if (fmt != BAT_KV_MXFP8 && fmt != BAT_KV_MXFP4) return BAT_ERR_INVALID_ARG;
  if (out_dtype != BAT_OUT_BF16 && out_dtype != BAT_OUT_F32) return BAT_ERR_INVALID_ARG;
  if (!cache_codes || !cache_scales || !slots || !out) return BAT_ERR_INVALID_ARG;
  if ((A == nullptr) != (B == nullptr)) return BAT_ERR_INVALID_ARG;
  if (!aligned16(cache_codes) || !aligned16(out) || (reinterpret_cast<uintptr_t>(slots) & 7u) != 0 ||
      (A && (!aligned16(A) || !aligned16(B))))
    return BAT_ERR_ALIGN;
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  bat::KvReadParams p;
  p.codes = static_cast<const uint8_t*>(cache_codes);
  p.scales = static_cast<const uint8_t*>(cache_scales);
  p.slots = slots;
  p.a = A;
  p.b = B;
  p.out = out;
  p.T = T;
  p.H = H;
  p.S = num_slots;
  p.D = static_cast<int>(D);
  p.nbh = static_cast<int>(D / 32);
  p.groups = (p.nbh + 3) / 4;
  p.ls = ls;
  const unsigned grid = kv_grid(T * H * p.groups, sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void (*k)(bat::KvReadParams);
  const bool fp8 = fmt == BAT_KV_MXFP8, xf = A != nullptr, f32 = out_dtype == BAT_OUT_F32;
  if (fp8)
    k = xf ? (f32 ? bat::bat_kv_dequantize_kernel<true, true, true> : bat::bat_kv_dequantize_kernel<true, true, false>)
           : (f32 ? bat::bat_kv_dequantize_kernel<true, false, true> : bat::bat_kv_dequantize_kernel<true, false, false>);
  else
    k = xf ? (f32 ? bat::bat_kv_dequantize_kernel<false, true, true> : bat::bat_kv_dequantize_kernel<false, true, false>)
           : (f32 ? bat::bat_kv_dequantize_kernel<false, false, true> : bat::bat_kv_dequantize_kernel<false, false, false>);
  k<<<grid, bat::kv::kThreads, 0, s>>>(p);
  return cuda_status(cudaGetLastError());
}

bat_status_t bat_w4a8_gemm(const bat_mxfp8_t* Xq, const bat_mxfp4_t* Wq, void* Y,
                           bat_out_dtype_t out_dtype, void* stream) {
  bat_status_t st = check_gemm_args(Xq, Wq, Y, out_dtype, true);
  if (st != BAT_OK) return st;
  return launch_gemm(Xq, Wq, Y, out_dtype, static_cast<cudaStream_t>(stream), true);
}

size_t bat_linear_workspace_bytes(int64_t M, int64_t K) {
  const size_t c = bat_mxfp4_codes_bytes(M, K);
  const size_t s = bat_mxfp4_scales_bytes(M, K);
  if (!c || !s) return 0;
  // decode sizes (row quantizer): the quantizer's completion flags after the scales
  if (M <= kRowsCudaCore)
    return static_cast<size_t>(round_up(static_cast<int64_t>(c), 256) +
                               round_up(static_cast<int64_t>(s), 256)) + kDoneFlagBytes;
  // CTA-pair GEMM sizes: the prologue's per-CTA completion flags (fused)
  if (M > 128)
    return static_cast<size_t>(round_up(static_cast<int64_t>(c), 256) +
                               round_up(static_cast<int64_t>(s), 256)) + kDoneFlagBytes;
  return static_cast<size_t>(round_up(static_cast<int64_t>(c), 256)) + s;
}

bat_status_t bat_linear(const void* X, int64_t M, const bat_mxfp4_t* Wq, const float* A,
                        const float* B, const float* g_lo, const float* g_hi, void* Y,
                        bat_out_dtype_t out_dtype, void* workspace, size_t workspace_bytes,
                        int fused, void* stream) {
  if (!Wq || (fused != 0 && fused != 1)) return BAT_ERR_INVALID_ARG;
  const int64_t K = Wq->k;
  if (M < 1 || K < 32) return BAT_ERR_INVALID_ARG;
  if (K % 32 != 0 || K > kMaxK || M > kMaxRows) return BAT_ERR_SHAPE;
  const size_t need = bat_linear_workspace_bytes(M, K);
  if (!workspace || workspace_bytes < need) return BAT_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BAT_ERR_ALIGN;
  bat_mxfp4_t xq;
  xq.codes = workspace;
  xq.scales = static_cast<uint8_t*>(workspace) + round_up(static_cast<int64_t>(bat_mxfp4_codes_bytes(M, K)), 256);
  xq.rows = M;
  xq.k = K;
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, &xq);
  if (st != BAT_OK) return st;
  st = check_gemm_args(&xq, Wq, Y, out_dtype);
  if (st != BAT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // decode sizes: the row quantizer signals completion through flags after the scales,
  // which the GEMM waits on (see launch_gemm)
  unsigned long long* flags = nullptr;
  unsigned long long epoch = 0;
  int q_ctas = 0;
  // fused (more than 128 rows): the prologue publishes each (token tile, block pair) as
  // it is stored and the CTA-pair GEMM waits for its token tiles only
  unsigned long long* cta_flags = nullptr;
  int q_strips = 0, q_cps = 0;
  uint8_t* after_scales = static_cast<uint8_t*>(xq.scales) +
                          round_up(static_cast<int64_t>(bat_mxfp4_scales_bytes(M, K)), 256);
  if (M <= kRowsCudaCore) {
    flags = reinterpret_cast<unsigned long long*>(after_scales);
    epoch = next_epoch();
  } else if (fused && M > 128) {
    cta_flags = reinterpret_cast<unsigned long long*>(after_scales);
    epoch = next_epoch();
  }
  st = launch_prologue(X, M, K, A, B, g_lo, g_hi, false, &xq, nullptr, s, 3, false, nullptr, 0, 0,
                       flags, epoch, &q_ctas, cta_flags, &q_strips, &q_cps);
  if (st != BAT_OK) return st;
  // the kernel right before the GEMM is the quantizer, which does not write the weights
  return launch_gemm(&xq, Wq, Y, out_dtype, s, false, true, flags, q_ctas, epoch, cta_flags,
                     q_strips, q_cps);
}

const char* bat_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(t_last_cuda_error);
}

int bat_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, bat::g_dev_error, sizeof(v)) != cudaSuccess) return -1;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(bat::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
  return static_cast<int>(v);
}

}  // extern "C"

// ---------------------------------------------------------------- bounded-wait self-test
namespace bat {
// One thread waits on an mbarrier that nothing arrives on, with the kernels' bounded
// wait pattern but the caller's limit; when the limit runs out it records
// kErrWaitFull in the device error word and returns (no trap, no endless spin).
__global__ void bat_selftest_wait_kernel(uint64_t limit_ns, unsigned int* waited_out) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!done) {
    if (mbar_try_wait_sleep(b, 0, 100000u)) break;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_dev_error, kErrWaitFull);
      done = true;
    }
  }
  *waited_out = done ? 1u : 0u;
  mbar_arrive(b);  // complete the phase before the barrier's memory goes away
}
}  // namespace bat

extern "C" bat_status_t bat_selftest_bounded_wait(uint64_t limit_ns, unsigned int* waited_out,
                                                  void* stream) {
  if (!waited_out || limit_ns == 0 || limit_ns > 2000000000ull) return BAT_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  bat::bat_selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, waited_out);
  return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------- element conversion
namespace bat {
__global__ void bat_e2m1_encode_kernel(const float* v, int64_t n, uint8_t* codes) {
  // Pairs (2t, 2t+1) go through the same conversion as the prologue (2t in the
  // low nibble); each code is returned in its own byte (sign in bit 3).
  const int64_t pairs = (n + 1) / 2;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < pairs;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float lo = v[2 * t];
    const float hi = (2 * t + 1 < n) ? v[2 * t + 1] : 0.0f;
    const uint32_t byte = e2m1x2(lo, hi);
    codes[2 * t] = static_cast<uint8_t>(byte & 0xFu);
    if (2 * t + 1 < n) codes[2 * t + 1] = static_cast<uint8_t>(byte >> 4);
  }
}
__global__ void bat_e4m3_encode_kernel(const float* v, int64_t n, uint8_t* codes) {
  // Groups (4t .. 4t+3) go through the conversion the MXFP8 prologue uses (4t in the
  // low byte); each code is returned in its own byte (sign in bit 7).
  const int64_t quads = (n + 3) / 4;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < quads;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float f[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = (4 * t + i < n) ? v[4 * t + i] : 0.0f;
    const uint32_t w = e4m3x4(f[0], f[1], f[2], f[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (4 * t + i < n) codes[4 * t + i] = static_cast<uint8_t>(w >> (8 * i));
  }
}
}  // namespace bat

extern "C" bat_status_t bat_e4m3_encode(const float* v, int64_t n, uint8_t* codes, void* stream) {
  if (!v || !codes || n < 1) return BAT_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  const int64_t blocks = ((n + 3) / 4 + 255) / 256;
  bat::bat_e4m3_encode_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0,
                                static_cast<cudaStream_t>(stream)>>>(v, n, codes);
  return cuda_status(cudaGetLastError());
}

extern "C" bat_status_t bat_e2m1_encode(const float* v, int64_t n, uint8_t* codes, void* stream) {
  if (!v || !codes || n < 1) return BAT_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  bat_status_t st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  int64_t blocks = ((n + 1) / 2 + 255) / 256;
  if (blocks > static_cast<int64_t>(sms) * 32) blocks = static_cast<int64_t>(sms) * 32;
  bat::bat_e2m1_encode_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                                static_cast<cudaStream_t>(stream)>>>(v, n, codes);
  return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------- allocation-free linear
// Scratch for bat_linear_noalloc: holds the quantized activations (codes, then
// tiled scales at a 256-byte boundary). Host code must not use this name as an
// address; the device address comes from cudaGetSymbolAddress per device.
static __device__ __align__(256) uint8_t bat_noalloc_scratch[BAT_NOALLOC_SCRATCH_BYTES];

namespace {
std::atomic<void*> g_noalloc_addr[64];

// Device address of the scratch array on the current device `dev` (looked up once).
bat_status_t noalloc_scratch(int dev, void** out) {
  void* p = g_noalloc_addr[dev].load();
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, bat_noalloc_scratch) != cudaSuccess || p == nullptr)
      return BAT_ERR_CUDA;
    g_noalloc_addr[dev].store(p);
  }
  *out = p;
  return BAT_OK;
}
}  // namespace

extern "C" bat_status_t bat_linear_noalloc(const void* X, int64_t M, const bat_mxfp4_t* Wq,
                                           const float* A, const float* B, const float* g_lo,
                                           const float* g_hi, void* Y, bat_out_dtype_t out_dtype,
                                           void* stream) {
  if (!Wq) return BAT_ERR_INVALID_ARG;
  const int64_t K = Wq->k;
  if (M < 1 || K < 32) return BAT_ERR_INVALID_ARG;
  if (K % 32 != 0 || K > kMaxK || M > kMaxRows) return BAT_ERR_SHAPE;
  const size_t need = bat_linear_workspace_bytes(M, K);
  if (need == 0 || need > BAT_NOALLOC_SCRATCH_BYTES) return BAT_ERR_WORKSPACE;
  bat_mxfp4_t xq;
  xq.codes = nullptr;  // placeholder until the device address is known
  xq.scales = nullptr;
  xq.rows = M;
  xq.k = K;
  // Validate with stand-in aligned addresses first, so bad arguments launch nothing.
  bat_mxfp4_t probe = xq;
  probe.codes = reinterpret_cast<void*>(static_cast<uintptr_t>(256));
  probe.scales = reinterpret_cast<void*>(static_cast<uintptr_t>(512));
  bat_status_t st = check_act_args(X, M, K, A, B, g_lo, g_hi, &probe);
  if (st != BAT_OK) return st;
  st = check_gemm_args(&probe, Wq, Y, out_dtype);
  if (st != BAT_OK) return st;
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != BAT_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(dev, &scratch);
  if (st != BAT_OK) return st;
  xq.codes = scratch;
  xq.scales = static_cast<uint8_t*>(scratch) +
              round_up(static_cast<int64_t>(bat_mxfp4_codes_bytes(M, K)), 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // decode sizes: the row quantizer signals completion through flags after the scales,
  // which the GEMM waits on (see launch_gemm)
  unsigned long long* flags = nullptr;
  unsigned long long epoch = 0;
  int q_ctas = 0;
  if (M <= kRowsCudaCore) {
    flags = reinterpret_cast<unsigned long long*>(
        static_cast<uint8_t*>(xq.scales) +
        round_up(static_cast<int64_t>(bat_mxfp4_scales_bytes(M, K)), 256));
    epoch = next_epoch();
  }
  st = launch_prologue(X, M, K, A, B, g_lo, g_hi, false, &xq, nullptr, s, 3, false, nullptr, 0, 0,
                       flags, epoch, &q_ctas);
  if (st != BAT_OK) return st;
  // the kernel right before the GEMM is the quantizer, which does not write the weights
  return launch_gemm(&xq, Wq, Y, out_dtype, s, false, true, flags, q_ctas, epoch);
}
