// The C ABI of libttq.so (declared in include/ttq.h): argument checks,
// workspace layout, TMA descriptor set-up and the order of the kernels of
// one TTQ linear call.  Nothing here allocates device memory or
// synchronises; every call only enqueues work on the caller's stream.
#include <atomic>
#include <cmath>
#include <mutex>

#include "ttq.h"
#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr size_t kAlign = 256;
// Workspace header, zeroed by ttq_workspace_init and left at zero by every
// call: word 0 the flags; words 64..1023 one counter per column block of the
// statistic pass (merge tickets / barrier counts); bytes 4096..20479 one
// arrival ticket per 128-row tile of the single-pass decode product.
constexpr size_t kStatusBytes = 4096;           // the least workspace an entry point takes
constexpr size_t kTicketsOffset = 4096;
constexpr size_t kHeaderBytes = kTicketsOffset + 4 * static_cast<size_t>(kFusedDecodeMaxTiles);
constexpr int64_t kMaxColumnBlocks = 960;       // tickets after the first 256 bytes
constexpr int kPlanSMs = 148;                   // fixed so the layout is device-independent

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms() {
  static std::atomic<int> cache[64] = {};   // host threads that race here store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return kPlanSMs;
  if (dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = kPlanSMs;
  if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool valid_qparams(int bits, int group) {
  return ((bits >= 2 && bits <= 4) || bits == 8) &&
         (group == 32 || group == 64 || group == 128 || group == 256);
}

// Whether a code scheme takes this bit width: the INT schemes 2..4 bits,
// FP8 (E4M3) exactly 8.
bool scheme_bits_ok(ttq_qscheme scheme, int bits) {
  return scheme == TTQ_QSCHEME_FP8_E4M3 ? bits == 8 : (bits >= 2 && bits <= 4);
}

// Whether ttq_linear_forward materialises the dequantised weight s (q - z)
// in binary16 and runs the product on it (more than one 256-token tile:
// dequantising inside the product would repeat the work once per tile)
// instead of dequantising the codes inside the product.
// 8-bit (FP8) codes are always materialised: no product reads them.
bool decode_reads_fp8(int64_t d, int64_t T) { return T <= 16 && d % 64 == 0; }
bool materialize_w(int64_t dp, int64_t T, int bits, int64_t d) {
  return dp > 0 && (T > 256 || (bits == 8 && !decode_reads_fp8(d, T)));
}

// Whether ttq_linear_forward takes the single-pass decode product (W read
// once, quantised and multiplied in one kernel, no codes written) for this
// shape: bf16 layers with the asymmetric INT codes and at most 16 tokens.
bool single_pass_decode(ttq_dtype dtype, ttq_qscheme scheme, int64_t d, int64_t dp, int64_t T,
                        int bits, int group) {
  return dtype == TTQ_BF16 && scheme == TTQ_QSCHEME_ASYMMETRIC &&
         fused_decode_supported(dp, d, T, bits, group);
}

// Computes the workspace layout; false for an unsupported shape.
// The plan of the product on the materialised weight: K splits only for
// more than 256 tokens, planned for 148 SMs whatever the device so that the
// workspace layout does not depend on it.
GemmPlan product_plan(int64_t dp, int64_t T, int64_t d, int64_t r, bool allow_split) {
  return gemm_plan_plain(dp, T, d, r, kPlanSMs, allow_split && T > 256);
}

// The number of parts of the low-rank A X product's reduction over d
// (1: none): the warp-level MMA kernel's channel slices for 17 to 512
// tokens, else the tensor-core GEMM's K splits.
int ax_parts(int64_t r, int64_t T, int64_t d) {
  const AxMmaPlan mp = ax_mma_plan(r, T, d);
  return mp.splits > 0 ? mp.splits : ax_split_plan(r, T, d, kPlanSMs).splits;
}

bool make_layout(int64_t d, int64_t dp, int64_t T, int64_t r, int bits, int group,
                 ttq_dtype dtype, ttq_workspace_layout* L) {
  if (d < 8 || d % 8 != 0 || dp < 0 || T < 0 || r < 0 || r % 8 != 0) return false;
  if ((d + 255) / 256 > kMaxColumnBlocks) return false;
  const bool has_q = dp > 0;
  if (has_q && (!valid_qparams(bits, group) || d % group != 0)) return false;
  if (dtype != TTQ_F32 && dtype != TTQ_BF16 && dtype != TTQ_F16) return false;
  ttq_workspace_layout l = {};
  int64_t splits = 1, rps = 1;
  act_norm_plan(d, T, kPlanSMs, &splits, &rps);
  size_t off = 0;
  l.status = off;
  off += kHeaderBytes;
  l.D = off;
  off = align_up(off + 4 * static_cast<size_t>(d));
  l.D_rsqrt = off;
  off = align_up(off + 4 * static_cast<size_t>(d));
  l.partial = off;
  off = align_up(off + 8 * static_cast<size_t>(splits) * static_cast<size_t>(d));
  if (has_q) {
    l.codes = off;
    off = align_up(off + static_cast<size_t>(dp) * static_cast<size_t>(d * bits / 32) * 4);
    l.scales = off;
    off = align_up(off + static_cast<size_t>(dp) * static_cast<size_t>(d / group) * 2);
    l.zeros = off;
    off = align_up(off + static_cast<size_t>(dp) * static_cast<size_t>(d / group) * 2);
  }
  l.ax_ld = 0;
  l.ax_splits = 0;
  if (r > 0) {
    l.ax_ld = r;
    l.ax = off;
    off = align_up(off + static_cast<size_t>(T) * static_cast<size_t>(r) * 2);
    const int parts = ax_parts(r, T, d);
    l.ax_splits = parts;
    if (parts > 1) {
      l.axp = off;
      off = align_up(off + static_cast<size_t>(parts) * static_cast<size_t>(T) *
                               static_cast<size_t>(r) * 4);
    }
  }
  if (has_q && dtype == TTQ_BF16 && fused_decode_supported(dp, d, T, bits, group)) {
    // the single-pass decode product: sqrt(D), its partial tiles and tickets
    l.D_sqrt = off;
    off = align_up(off + 4 * static_cast<size_t>(d));
    l.ypart = off;
    off = align_up(off + 4 * static_cast<size_t>(fused_decode_plan(dp, d, T).part_floats));
    l.tickets = kTicketsOffset;
  }
  if (has_q) {
    l.xh = off;
    off = align_up(off + static_cast<size_t>(T) * static_cast<size_t>(d) * 2);
  }
  if (dtype == TTQ_F32 && r > 0) {
    l.xb = off;
    off = align_up(off + static_cast<size_t>(T) * static_cast<size_t>(d) * 2);
    l.ab = off;
    off = align_up(off + (static_cast<size_t>(r) * d + static_cast<size_t>(dp) * r) * 2);
  }
  if (has_q && materialize_w(dp, T, bits, d)) {
    l.wq = off;
    off = align_up(off + static_cast<size_t>(dp) * static_cast<size_t>(d) * 2);
    // the product on W_hat split along K: its float32 partial sums
    const GemmPlan plan = product_plan(dp, T, d, r, true);
    if (plan.splits > 1) {
      l.ypart = off;
      off = align_up(off + static_cast<size_t>(plan.splits) * static_cast<size_t>(T) *
                               static_cast<size_t>(dp) * 4);
    }
  }
  l.total = off;
  l.splits = splits;
  *L = l;
  return true;
}

// ----------------------------------------------------- tensor map encoding
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// 16-bit matrix [outer][inner] (bf16 or binary16) with row stride ld
// (elements), loaded as box_outer rows x 64 columns into the
// 128-byte-swizzled layout; reads outside the matrix return zeros.
bool encode_16bit(CUtensorMap* m, const void* base, bool f16, int64_t inner, int64_t outer,
                  int64_t ld, int box_outer) {
  EncodeFn enc = get_encode();
  if (enc == nullptr || inner < 1 || outer < 1) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_outer)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed codes [rows][wpr] as uint32, loaded as box_rows x box_words tiles
// without swizzle.  The row stride must be a multiple of 16 bytes.
bool encode_codes(CUtensorMap* m, const uint32_t* base, int64_t wpr, int64_t rows, int box_words,
                  int box_rows) {
  EncodeFn enc = get_encode();
  if (enc == nullptr || wpr < 1 || rows < 1 || (wpr * 4) % 16 != 0) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(wpr) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_words), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 3-D view of a dense buffer: dims[0] innermost (element stride 1),
// strides (bytes) of dims 1 and 2 in any order, reads outside the view
// return zeros.
bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType type, const int64_t (&dims)[3],
               const int64_t (&strides)[2], const int (&box)[3], CUtensorMapSwizzle swizzle) {
  EncodeFn enc = get_encode();
  if (enc == nullptr) return false;
  for (int i = 0; i < 3; ++i)
    if (dims[i] < 1 || box[i] < 1 || box[i] > 256) return false;
  for (int i = 0; i < 2; ++i)
    if (strides[i] % 16 != 0) return false;
  const cuuint64_t gd[3] = {static_cast<cuuint64_t>(dims[0]), static_cast<cuuint64_t>(dims[1]),
                            static_cast<cuuint64_t>(dims[2])};
  const cuuint64_t gs[2] = {static_cast<cuuint64_t>(strides[0]), static_cast<cuuint64_t>(strides[1])};
  const cuuint32_t bx[3] = {static_cast<cuuint32_t>(box[0]), static_cast<cuuint32_t>(box[1]),
                            static_cast<cuuint32_t>(box[2])};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, type, 3, const_cast<void*>(base), gd, gs, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 Y [rows][cols] (row stride cols), stored as box_rows x box_cols tiles
// without swizzle.
bool encode_y_bf16(CUtensorMap* m, void* base, int64_t cols, int64_t rows, int box_cols,
                   int box_rows) {
  EncodeFn enc = get_encode();
  if (enc == nullptr || cols < 1 || rows < 1 || (cols * 2) % 16 != 0) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

ttq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TTQ_OK : TTQ_ERR_CUDA; }

uint8_t* ws_at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// A X [T][r] bf16 into the workspace: the plain-operand mode of the GEMM
// (M = r rows of A), split along K when its few output tiles would leave
// most SMs idle (float32 partials, then a reduction in split order).
ttq_status run_ax(const void* Ab, const void* Xb, int64_t d, int64_t T, int64_t r, void* ws,
                  const ttq_workspace_layout& L, cudaStream_t stream, bool pdl) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  void* ax = ws_at(ws, L.ax);
  const AxMmaPlan mp = ax_mma_plan(r, T, d);
  if (mp.splits > 0) {
    // 17 to 512 tokens: warp-level MMAs over channel slices
    const bool split = mp.splits > 1;
    if (split && (L.axp == 0 || L.ax_splits != mp.splits)) return TTQ_ERR_WORKSPACE;
    float* P = split ? reinterpret_cast<float*>(ws_at(ws, L.axp)) : nullptr;
    const ttq_status st =
        cuda_status(launch_ax_mma(Ab, Xb, d, T, r, mp, P, ax, L.ax_ld, stream, pdl));
    if (st != TTQ_OK || !split) return st;
    return cuda_status(launch_ax_reduce(P, mp.splits, T, r, ax, L.ax_ld, stream, true));
  }
  const int bn = gemm_block_n(T);
  GemmMaps m;
  if (!encode_16bit(&m.a0, Ab, false, d, r, d, 128) || !encode_16bit(&m.b0, Xb, false, d, T, d, bn))
    return TTQ_ERR_CUDA;
  m.a1 = m.a0;
  m.b1 = m.b0;
  m.c0 = m.b0;
  m.y = m.b0;
  GemmArgs a;
  a.bits = 0;
  a.K = d;
  a.M = r;
  a.T = T;
  a.K_tail = 0;
  a.status = status;
  const AxSplit sp = ax_split_plan(r, T, d, kPlanSMs);
  if (sp.splits > 1 && L.axp != 0 && L.ax_splits == sp.splits) {
    float* P = reinterpret_cast<float*>(ws_at(ws, L.axp));
    a.Y = P;
    a.ldy = r;
    a.y_f32 = true;
    a.k_splits = sp.splits;
    a.kb_per_split = sp.kb_per_split;
    a.split_stride = T * r;
    ttq_status st = cuda_status(launch_dequant_gemm(a, m, bn, 128, stream, pdl));
    if (st != TTQ_OK) return st;
    return cuda_status(launch_ax_reduce(P, sp.splits, T, r, ax, L.ax_ld, stream, true));
  }
  a.Y = ax;
  a.ldy = L.ax_ld;
  a.y_f32 = false;
  return cuda_status(launch_dequant_gemm(a, m, bn, 128, stream, pdl));
}

// Y = W_hat X (+ B (A X)) from quantised weights.  Xh is binary16
// X D^(-1/2); Xb, Ab, Bb are bf16 X, A, B (used only when r > 0).
ttq_status run_gemm(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros,
                    const void* Xh, const void* Xb, const void* Ab,
                    const void* Bb, int64_t d, int64_t dp, int64_t T, int64_t r, int bits,
                    int group, void* Y, bool y_f32, void* ws, const ttq_workspace_layout& L,
                    cudaStream_t stream, bool pdl, const void* wq = nullptr,
                    float* ypart = nullptr) {
  if (T == 0 || dp == 0) return TTQ_OK;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  void* ax = r > 0 ? ws_at(ws, L.ax) : nullptr;
  if (r > 0) {
    const ttq_status st = run_ax(Ab, Xb, d, T, r, ws, L, stream, pdl);
    if (st != TTQ_OK) return st;
    pdl = true;
  }
  if (!wq && T <= 16) {
    // a few tokens: the product is bound by turning code bytes into
    // operands; they stream through shared memory in large stages and are
    // dequantised in registers for warp-level MMAs (when the shape allows
    // the unit-major views below)
    const DecodeMapShape sh = decode_map_shape(bits, static_cast<int>(T));
    const int64_t wpr = d * bits / 32;
    CUtensorMap tmC, tmX;
    if (d % (sh.unit_k * (bits == 3 ? 2 : 1)) == 0 && wpr % sh.piece_words == 0 &&
        encode_3d(&tmC, codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, {sh.piece_words, dp, wpr / sh.piece_words},
                  {wpr * 4, int64_t{sh.piece_words} * 4}, {sh.piece_words, sh.code_rows, sh.code_pieces},
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_3d(&tmX, Xh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, {sh.unit_k, T, d / sh.unit_k},
                  {d * 2, int64_t{sh.unit_k} * 2}, {sh.unit_k, sh.x_tokens, sh.x_units},
                  CU_TENSOR_MAP_SWIZZLE_128B)) {
      DecodeArgs a;
      a.scales = scales;
      a.zeros = zeros;
      a.K = d;
      a.M = dp;
      a.T = T;
      a.bits = bits;
      a.group = group;
      a.Blr = Bb;
      a.AX = ax;
      a.r = r;
      a.ax_ld = L.ax_ld;
      a.Y = Y;
      a.ldy = dp;
      a.y_f32 = y_f32;
      a.status = status;
      return cuda_status(launch_decode_gemm(a, tmC, tmX, stream, pdl));
    }
  }
  if (!wq && bits == 8) return TTQ_ERR_UNSUPPORTED;  // no other product reads 8-bit codes
  // wq: the product reads the materialised binary16 s (q - z) by TMA, split
  // along K where its plan says so and ypart has room for the partial sums
  int bm = 128, bnm = 16;
  GemmPlan plan{128, 16, 1, 0};
  if (wq) {
    plan = product_plan(dp, T, d, r, ypart != nullptr);
    bm = plan.block_m;
    bnm = plan.block_n;
  } else {
    gemm_tile_shape(bits, dp, T, device_sms(), &bm, &bnm);
  }
  const bool k_split = plan.splits > 1;
  GemmMaps m;
  if (!encode_16bit(&m.b0, Xh, true, d, T, d, bnm)) return TTQ_ERR_CUDA;
  m.a0 = m.b0;
  if (wq && !encode_16bit(&m.a0, wq, true, d, dp, d, bm)) return TTQ_ERR_CUDA;
  if (r > 0) {
    if (!encode_16bit(&m.a1, Bb, false, r, dp, r, bm) ||
        !encode_16bit(&m.b1, ax, false, r, T, L.ax_ld, bnm))
      return TTQ_ERR_CUDA;
  } else {
    m.a1 = m.b0;
    m.b1 = m.b0;
  }
  // the code tile comes in by TMA when the code rows are 16-byte strided
  const int64_t wpr = d * bits / 32;
  const bool codes_tma =
      !wq && encode_codes(&m.c0, codes, wpr, dp, gemm_code_tile_words(bits), bm);
  if (!codes_tma) m.c0 = m.b0;
  // bf16 Y goes out through TMA stores of 32 x 16 slabs when its rows are
  // 16-byte strided
  const bool y_tma = !k_split && !y_f32 && dp % 8 == 0 && encode_y_bf16(&m.y, Y, dp, T, 32, 16);
  if (!y_tma) m.y = m.b0;
  GemmArgs a;
  a.codes_tma = codes_tma;
  a.y_tma = y_tma;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.bits = wq ? 0 : bits;
  a.a_f16 = wq != nullptr;
  a.group = group;
  a.K = d;
  a.M = dp;
  a.T = T;
  a.K_tail = r;
  a.Y = k_split ? static_cast<void*>(ypart) : Y;
  a.ldy = dp;
  a.y_f32 = y_f32 || k_split;
  a.status = status;
  if (k_split) {
    a.k_splits = plan.splits;
    a.kb_per_split = plan.kb_per_split;
    a.split_stride = T * dp;
  }
  const ttq_status st = cuda_status(launch_dequant_gemm(a, m, bnm, bm, stream, pdl));
  if (st != TTQ_OK || !k_split) return st;
  return cuda_status(launch_y_reduce(ypart, plan.splits, T * dp, Y, y_f32, stream, true));
}

// Steps (2)-(3) in one pass over bf16 W (T <= 16): sqrt(D) in Dh, binary16
// X D^(-1/2) in Xh; codes/scales/zeros stored when codes is non-null.
ttq_status run_single_pass(const void* W, const float* Dh, const void* Xh, const void* Xb,
                           const void* Ab, const void* Bb, int64_t d, int64_t dp, int64_t T,
                           int64_t r, int bits, int group, uint32_t* codes, uint16_t* scales,
                           uint16_t* zeros, void* Y, bool y_f32, void* ws,
                           const ttq_workspace_layout& L, cudaStream_t stream, bool pdl) {
  if (T == 0 || dp == 0) return TTQ_OK;
  if (r > 0) {
    const ttq_status st = run_ax(Ab, Xb, d, T, r, ws, L, stream, pdl);
    if (st != TTQ_OK) return st;
    pdl = true;
  }
  CUtensorMap tmW, tmX;
  if (!encode_16bit(&tmW, W, false, d, dp, d, fused_decode_rows()) ||
      !encode_16bit(&tmX, Xh, true, d, T, d, T <= 8 ? 8 : 16))
    return TTQ_ERR_CUDA;
  FusedDecodeArgs a;
  a.Dh = Dh;
  a.K = d;
  a.M = dp;
  a.T = T;
  a.bits = bits;
  a.group = group;
  a.Blr = Bb;
  a.AX = r > 0 ? ws_at(ws, L.ax) : nullptr;
  a.r = r;
  a.ax_ld = L.ax_ld;
  a.Y = Y;
  a.ldy = dp;
  a.y_f32 = y_f32;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.part = reinterpret_cast<float*>(ws_at(ws, L.ypart));
  a.tickets = reinterpret_cast<uint32_t*>(ws_at(ws, L.tickets));
  a.status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  return cuda_status(launch_fused_decode(a, tmW, tmX, stream, pdl));
}

// Step (1) and, when xh is non-null, the product's binary16 operand
// X D^(-1/2) in xh: one fused kernel (the splits of a column block form a
// thread-block cluster) when each split's rows fit in registers, else the
// statistic kernel followed by the scaling kernel.  Either way D and D_rsqrt
// are the same bits (same splits, same merge order).  xb: bf16 copy of a
// float32 X (or null).
ttq_status run_statistic(const void* X, ttq_dtype dtype, int64_t d, int64_t T, float p,
                         float lambda, float alpha, const ttq_workspace_layout& L, void* ws,
                         float* D, float* Dr, void* xh, void* xb, cudaStream_t s,
                         float* Dh = nullptr) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  double* partial = reinterpret_cast<double*>(ws_at(ws, L.partial));
  const bool f32 = dtype == TTQ_F32;
  int64_t splits, rps;
  act_norm_plan(d, T, kPlanSMs, &splits, &rps);
  if (xh != nullptr) {
    bool fused = false;
    const ttq_status st = cuda_status(launch_act_norm_scale(X, f32, d, T, p, lambda, alpha,
                                                            splits, rps, D, Dr, xh, xb, status, s,
                                                            &fused, Dh));
    if (st != TTQ_OK || fused) return st;
  }
  ttq_status st = cuda_status(launch_act_norm(X, f32, d, T, p, lambda, alpha, splits, rps,
                                              partial, status + 64, D, Dr, nullptr, xb, status,
                                              s, false, Dh));
  if (st != TTQ_OK || xh == nullptr) return st;
  return cuda_status(launch_scale_to_f16(X, dtype, Dr, xh, T, d, status, device_sms(), s, true));
}

}  // namespace

bool encode_bf16_box(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int box_cols,
                     int box_rows) {
  EncodeFn enc = get_encode();
  if (enc == nullptr || cols < 1 || rows < 1 || (cols * 2) % 16 != 0 || box_cols < 8 ||
      box_cols > 256 || (box_cols * 2) % 16 != 0 || box_rows < 1 || box_rows > 256 ||
      (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ttq

using namespace ttq;

extern "C" {

size_t ttq_workspace_size(int64_t d, int64_t dp, int64_t T, int64_t r, int bits, int group,
                          ttq_dtype dtype) {
  ttq_workspace_layout L;
  if (!make_layout(d, dp, T, r, bits, group, dtype, &L)) return 0;
  return L.total;
}

ttq_status ttq_workspace_get_layout(int64_t d, int64_t dp, int64_t T, int64_t r, int bits,
                                    int group, ttq_dtype dtype, ttq_workspace_layout* out) {
  if (out == nullptr) return TTQ_ERR_INVALID_ARG;
  if (!make_layout(d, dp, T, r, bits, group, dtype, out)) return TTQ_ERR_INVALID_ARG;
  return TTQ_OK;
}

ttq_status ttq_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return TTQ_ERR_INVALID_ARG;
  const size_t n = ws_bytes < kHeaderBytes ? ws_bytes : kHeaderBytes;
  return cuda_status(cudaMemsetAsync(ws, 0, n, static_cast<cudaStream_t>(stream)));
}

ttq_status ttq_act_norm(const void* X, ttq_dtype dtype, int64_t d, int64_t T, float p,
                        float lambda, float alpha, float* D, float* D_rsqrt, void* ws,
                        size_t ws_bytes, void* stream) {
  if (dtype == TTQ_F16) return TTQ_ERR_INVALID_ARG;
  ttq_workspace_layout L;
  if (!make_layout(d, 0, T, 0, 4, 32, dtype, &L)) return TTQ_ERR_INVALID_ARG;
  if ((T > 0 && X == nullptr) || ws == nullptr || !(p >= 1.0f) || !(lambda >= 0.0f) ||
      !(alpha >= 0.0f) || !std::isfinite(p) || !std::isfinite(lambda) || !std::isfinite(alpha))
    return TTQ_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (D && !aligned16(D)) || (D_rsqrt && !aligned16(D_rsqrt)) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return TTQ_ERR_INVALID_ARG;
  const size_t need = L.partial + align_up(8 * static_cast<size_t>(L.splits) * d);
  if (ws_bytes < need) return TTQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  float* Dw = reinterpret_cast<float*>(ws_at(ws, L.D));
  float* Drw = reinterpret_cast<float*>(ws_at(ws, L.D_rsqrt));
  int64_t splits, rps;
  act_norm_plan(d, T, kPlanSMs, &splits, &rps);
  ttq_status st = cuda_status(launch_act_norm(
      X, dtype == TTQ_F32, d, T, p, lambda, alpha, splits, rps,
      reinterpret_cast<double*>(ws_at(ws, L.partial)), status + 64, Dw, Drw, nullptr, nullptr,
      status, s));
  if (st != TTQ_OK) return st;
  if (D) st = cuda_status(cudaMemcpyAsync(D, Dw, 4 * d, cudaMemcpyDeviceToDevice, s));
  if (st == TTQ_OK && D_rsqrt)
    st = cuda_status(cudaMemcpyAsync(D_rsqrt, Drw, 4 * d, cudaMemcpyDeviceToDevice, s));
  return st;
}

ttq_status ttq_act_norm_scale(const void* X, ttq_dtype dtype, int64_t d, int64_t T, float p,
                              float lambda, float alpha, float* D, float* D_rsqrt, uint16_t* Xs,
                              void* ws, size_t ws_bytes, void* stream) {
  if (dtype == TTQ_F16) return TTQ_ERR_INVALID_ARG;
  ttq_workspace_layout L;
  if (!make_layout(d, 0, T, 0, 4, 32, dtype, &L)) return TTQ_ERR_INVALID_ARG;
  if ((T > 0 && (X == nullptr || Xs == nullptr)) || ws == nullptr || !(p >= 1.0f) ||
      !(lambda >= 0.0f) || !(alpha >= 0.0f) || !std::isfinite(p) || !std::isfinite(lambda) ||
      !std::isfinite(alpha))
    return TTQ_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (Xs && !aligned16(Xs)) || (D && !aligned16(D)) ||
      (D_rsqrt && !aligned16(D_rsqrt)) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return TTQ_ERR_INVALID_ARG;
  const size_t need = L.partial + align_up(8 * static_cast<size_t>(L.splits) * d);
  if (ws_bytes < need) return TTQ_ERR_WORKSPACE;
  float* Dw = D ? D : reinterpret_cast<float*>(ws_at(ws, L.D));
  float* Drw = D_rsqrt ? D_rsqrt : reinterpret_cast<float*>(ws_at(ws, L.D_rsqrt));
  if (T == 0) Xs = nullptr;  // nothing to scale
  return run_statistic(X, dtype, d, T, p, lambda, alpha, L, ws, Dw, Drw, Xs, nullptr,
                       static_cast<cudaStream_t>(stream));
}

ttq_status ttq_linear_forward_kernels(ttq_dtype dtype, int64_t d, int64_t dp, int64_t T,
                                      int64_t r, float p, int bits, int group, ttq_qscheme scheme,
                                      int* kernels) {
  if (kernels == nullptr || (dtype != TTQ_F32 && dtype != TTQ_BF16)) return TTQ_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0 || dp < 0 || T < 0 || r < 0 || !(p >= 1.0f) || !std::isfinite(p))
    return TTQ_ERR_INVALID_ARG;
  if (scheme != TTQ_QSCHEME_ASYMMETRIC && scheme != TTQ_QSCHEME_SYMMETRIC &&
      scheme != TTQ_QSCHEME_FP8_E4M3)
    return TTQ_ERR_INVALID_ARG;
  int64_t splits, rps;
  act_norm_plan(d, T, kPlanSMs, &splits, &rps);
  const bool f32 = dtype == TTQ_F32;
  int n = 1;  // statistic
  if (dp > 0) {
    if (!act_norm_scale_fused(f32, splits, rps, p)) ++n;                  // separate scaling
    const bool one_pass = T > 0 && single_pass_decode(dtype, scheme, d, dp, T, bits, group);
    if (!one_pass) ++n;                                                    // quantiser
    if (T > 0) {
      ++n;                                                                 // product
      if (materialize_w(dp, T, bits, d) && product_plan(dp, T, d, r, true).splits > 1)
        ++n;                                                               // its split reduction
      if (r > 0) {
        n += 1 + (f32 ? 2 : 0);                                            // A X (+ bf16 A, B)
        if (ax_parts(r, T, d) > 1) ++n;                                    // its split reduction
      }
    }
  }
  *kernels = n;
  return TTQ_OK;
}

ttq_status ttq_quantize_gemm(const void* W, const float* D, const uint16_t* Xs, const void* A,
                             const void* B, const void* X, int64_t d, int64_t dp, int64_t T,
                             int64_t r, int bits, int group, uint32_t* codes, uint16_t* scales,
                             uint16_t* zeros, void* Y, ttq_dtype y_dtype, void* ws,
                             size_t ws_bytes, void* stream) {
  if (y_dtype != TTQ_F32 && y_dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0 || dp < 0 || T < 0 || r < 0) return TTQ_ERR_INVALID_ARG;
  if (!valid_qparams(bits, group) || bits == 8 || d % group != 0) return TTQ_ERR_UNSUPPORTED;
  const bool work = dp > 0 && T > 0;
  if (work && !fused_decode_supported(dp, d, T, bits, group)) return TTQ_ERR_UNSUPPORTED;
  ttq_workspace_layout L;
  if (!make_layout(d, dp, T, r, bits, group, TTQ_BF16, &L)) return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  if (work && (W == nullptr || D == nullptr || Xs == nullptr || Y == nullptr))
    return TTQ_ERR_INVALID_ARG;
  if (r > 0 && (A == nullptr || B == nullptr || X == nullptr)) return TTQ_ERR_INVALID_ARG;
  if ((codes == nullptr) != (scales == nullptr) || (codes == nullptr) != (zeros == nullptr))
    return TTQ_ERR_INVALID_ARG;
  const void* ptrs[] = {W, D, Xs, A, B, X, codes, scales, zeros, Y};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return TTQ_ERR_INVALID_ARG;
  if (!work) return TTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* Dh = reinterpret_cast<float*>(ws_at(ws, L.D_sqrt));
  const ttq_status st = cuda_status(launch_sqrt_f32(D, Dh, d, s));
  if (st != TTQ_OK) return st;
  return run_single_pass(W, Dh, Xs, X, A, B, d, dp, T, r, bits, group, codes, scales, zeros, Y,
                         y_dtype == TTQ_F32, ws, L, s, true);
}

ttq_status ttq_quantize_weight_ex(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                                  const float* D, int bits, int group, ttq_qscheme scheme,
                                  uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                                  uint16_t* W_hat, void* ws, size_t ws_bytes, void* stream) {
  if (scheme != TTQ_QSCHEME_ASYMMETRIC && scheme != TTQ_QSCHEME_SYMMETRIC &&
      scheme != TTQ_QSCHEME_FP8_E4M3)
    return TTQ_ERR_INVALID_ARG;
  if (W_hat && !aligned16(W_hat)) return TTQ_ERR_INVALID_ARG;
  if (dtype != TTQ_F32 && dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (bits < 1 || bits > 8 || group < 1) return TTQ_ERR_INVALID_ARG;
  if (!valid_qparams(bits, group) || !scheme_bits_ok(scheme, bits)) return TTQ_ERR_UNSUPPORTED;
  if (d < group || d % group != 0 || dp < 0) return TTQ_ERR_INVALID_ARG;
  // the codes, scales and zeros are written together, or (with W_hat) all left out
  const bool no_codes = codes == nullptr && scales == nullptr && zeros == nullptr;
  if (dp > 0 && (W == nullptr || (no_codes ? W_hat == nullptr
                                           : (codes == nullptr || scales == nullptr ||
                                              zeros == nullptr))))
    return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if ((W && !aligned16(W)) || (D && !aligned16(D)) || (codes && !aligned16(codes)))
    return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return TTQ_ERR_WORKSPACE;
  if (scheme == TTQ_QSCHEME_FP8_E4M3)
    return cuda_status(launch_qdq_fp8(W, dtype == TTQ_F32, dp, d, D, group, codes, scales, zeros,
                                      static_cast<uint32_t*>(ws), device_sms(),
                                      static_cast<cudaStream_t>(stream), false, W_hat));
  return cuda_status(launch_qdq_pack(W, dtype == TTQ_F32, dp, d, D, bits, group, codes, scales,
                                     zeros, static_cast<uint32_t*>(ws), device_sms(),
                                     static_cast<cudaStream_t>(stream), false, W_hat,
                                     scheme == TTQ_QSCHEME_SYMMETRIC));
}

ttq_status ttq_quantize_weight(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                               const float* D, int bits, int group, uint32_t* codes,
                               uint16_t* scales, uint16_t* zeros, void* ws, size_t ws_bytes,
                               void* stream) {
  return ttq_quantize_weight_ex(W, dtype, dp, d, D, bits, group, TTQ_QSCHEME_ASYMMETRIC, codes,
                                scales, zeros, nullptr, ws, ws_bytes, stream);
}

ttq_status ttq_quantize_dequant_weight(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                                       const float* D, int bits, int group, uint32_t* codes,
                                       uint16_t* scales, uint16_t* zeros, uint16_t* W_hat,
                                       void* ws, size_t ws_bytes, void* stream) {
  if (dp > 0 && W_hat == nullptr) return TTQ_ERR_INVALID_ARG;
  return ttq_quantize_weight_ex(W, dtype, dp, d, D, bits, group, TTQ_QSCHEME_ASYMMETRIC, codes,
                                scales, zeros, W_hat, ws, ws_bytes, stream);
}

ttq_status ttq_dequantized_gemm(const uint16_t* W_hat, const uint16_t* Xs, int64_t d, int64_t dp,
                                int64_t T, void* Y, ttq_dtype y_dtype, void* ws, size_t ws_bytes,
                                void* stream) {
  if (y_dtype != TTQ_F32 && y_dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0 || dp < 0 || T < 0) return TTQ_ERR_INVALID_ARG;
  const bool work = dp > 0 && T > 0;
  if (work && (W_hat == nullptr || Xs == nullptr || Y == nullptr)) return TTQ_ERR_INVALID_ARG;
  const void* ptrs[] = {W_hat, Xs, Y};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return TTQ_ERR_WORKSPACE;
  if (!work) return TTQ_OK;
  ttq_workspace_layout L = {};  // the status word (offset 0); the partial sums after the header
  float* ypart = nullptr;
  if (ws_bytes >= ttq_dequantized_gemm_workspace_size(d, dp, T) &&
      product_plan(dp, T, d, 0, true).splits > 1)
    ypart = reinterpret_cast<float*>(ws_at(ws, kHeaderBytes));
  return run_gemm(nullptr, nullptr, nullptr, Xs, nullptr, nullptr, nullptr, d, dp, T, 0, 4, 32,
                  Y, y_dtype == TTQ_F32, ws, L, static_cast<cudaStream_t>(stream), false, W_hat,
                  ypart);
}

size_t ttq_dequantized_gemm_workspace_size(int64_t d, int64_t dp, int64_t T) {
  if (d < 8 || d % 8 != 0 || dp < 0 || T < 0) return 0;
  const GemmPlan plan = product_plan(dp, T, d, 0, true);
  if (dp == 0 || T == 0 || plan.splits < 2) return kStatusBytes;
  return kHeaderBytes + static_cast<size_t>(plan.splits) * static_cast<size_t>(T) *
                            static_cast<size_t>(dp) * 4;
}

ttq_status ttq_scale_activations(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                                 const float* D_rsqrt, uint16_t* Xs, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (dtype != TTQ_F32 && dtype != TTQ_BF16 && dtype != TTQ_F16) return TTQ_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0 || T < 0) return TTQ_ERR_INVALID_ARG;
  if (T > 0 && (X == nullptr || Xs == nullptr)) return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (Xs && !aligned16(Xs)) || (D_rsqrt && !aligned16(D_rsqrt)))
    return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return TTQ_ERR_WORKSPACE;
  return cuda_status(launch_scale_to_f16(X, dtype, D_rsqrt, Xs, T, d, static_cast<uint32_t*>(ws),
                                         device_sms(), static_cast<cudaStream_t>(stream)));
}

ttq_status ttq_dequant_gemm(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros,
                            const float* D_rsqrt, const void* X, const void* A, const void* B,
                            ttq_dtype dtype, int64_t d, int64_t dp, int64_t T, int64_t r,
                            int bits, int group, void* Y, ttq_dtype y_dtype, void* ws,
                            size_t ws_bytes, void* stream) {
  if (y_dtype != TTQ_F32 && y_dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (bits >= 1 && bits <= 8 && group >= 1 &&
      (!valid_qparams(bits, group) || (bits == 8 && !decode_reads_fp8(d, T))))
    return TTQ_ERR_UNSUPPORTED;   // 8-bit (FP8) codes: only the decode product reads them
  ttq_workspace_layout L;
  if (!make_layout(d, dp, T, r, bits, group, dtype, &L)) return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  const bool work = dp > 0 && T > 0;
  if (work && (codes == nullptr || scales == nullptr || zeros == nullptr || X == nullptr ||
               Y == nullptr))
    return TTQ_ERR_INVALID_ARG;
  if (r > 0 && (A == nullptr || B == nullptr)) return TTQ_ERR_INVALID_ARG;
  if (dtype == TTQ_F16 && r > 0) return TTQ_ERR_UNSUPPORTED;
  const void* ptrs[] = {codes, scales, zeros, D_rsqrt, X, A, B, Y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTQ_ERR_INVALID_ARG;
  if (!work) return TTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  const bool f32 = dtype == TTQ_F32;
  const void* xh = X;  // binary16 X D^{-1/2} given as is
  ttq_status st = TTQ_OK;
  bool pdl = false;    // the first kernel of the call waits for earlier work normally
  if (!(dtype == TTQ_F16 && D_rsqrt == nullptr)) {
    pdl = true;
    void* xs = ws_at(ws, L.xh);
    st = cuda_status(launch_scale_to_f16(X, dtype, D_rsqrt, xs, T, d, status, device_sms(), s));
    if (st != TTQ_OK) return st;
    xh = xs;
  }
  const void* Xb = X;
  const void* Ab = A;
  const void* Bb = B;
  if (f32 && r > 0) {
    void* xb = ws_at(ws, L.xb);
    void* ab = ws_at(ws, L.ab);
    void* bb = static_cast<uint8_t*>(ab) + static_cast<size_t>(r) * d * 2;
    st = cuda_status(launch_to_bf16(static_cast<const float*>(X), xb, T * d, s));
    if (st == TTQ_OK) st = cuda_status(launch_to_bf16(static_cast<const float*>(A), ab, r * d, s));
    if (st == TTQ_OK) st = cuda_status(launch_to_bf16(static_cast<const float*>(B), bb, dp * r, s));
    if (st != TTQ_OK) return st;
    Xb = xb;
    Ab = ab;
    Bb = bb;
  }
  return run_gemm(codes, scales, zeros, xh, Xb, Ab, Bb, d, dp, T, r, bits, group, Y,
                  y_dtype == TTQ_F32, ws, L, s, pdl);
}

ttq_status ttq_linear_forward_ex(const void* X, const void* W, const void* A, const void* B,
                                 ttq_dtype dtype, int64_t d, int64_t dp, int64_t T, int64_t r,
                                 float p, float lambda, float alpha, int bits, int group,
                                 ttq_qscheme scheme, void* Y, ttq_dtype y_dtype, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (y_dtype != TTQ_F32 && y_dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (scheme != TTQ_QSCHEME_ASYMMETRIC && scheme != TTQ_QSCHEME_SYMMETRIC &&
      scheme != TTQ_QSCHEME_FP8_E4M3)
    return TTQ_ERR_INVALID_ARG;
  if (bits >= 1 && bits <= 8 && group >= 1 &&
      (!valid_qparams(bits, group) || !scheme_bits_ok(scheme, bits)))
    return TTQ_ERR_UNSUPPORTED;
  if (dtype == TTQ_F16) return TTQ_ERR_INVALID_ARG;
  ttq_workspace_layout L;
  if (!make_layout(d, dp, T, r, bits, group, dtype, &L)) return TTQ_ERR_INVALID_ARG;
  if (dp == 0 && !valid_qparams(bits, group)) return TTQ_ERR_INVALID_ARG;
  if (!(p >= 1.0f) || !(lambda >= 0.0f) || !(alpha >= 0.0f) || !std::isfinite(p) ||
      !std::isfinite(lambda) || !std::isfinite(alpha))
    return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return TTQ_ERR_WORKSPACE;
  if ((T > 0 && X == nullptr) || (dp > 0 && W == nullptr) || (T > 0 && dp > 0 && Y == nullptr))
    return TTQ_ERR_INVALID_ARG;
  if (r > 0 && (A == nullptr || B == nullptr)) return TTQ_ERR_INVALID_ARG;
  const void* ptrs[] = {X, W, A, B, Y};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return TTQ_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws_at(ws, L.status));
  float* D = reinterpret_cast<float*>(ws_at(ws, L.D));
  float* Dr = reinterpret_cast<float*>(ws_at(ws, L.D_rsqrt));
  const bool f32 = dtype == TTQ_F32;
  void* xh = dp > 0 ? ws_at(ws, L.xh) : nullptr;
  void* xb = (f32 && r > 0) ? ws_at(ws, L.xb) : nullptr;

  // (1) D and D^{-1/2} (a float32 X is also written as bf16 for the
  // low-rank product), then the product's B operand X D^{-1/2} in binary16
  const bool one_pass = T > 0 && single_pass_decode(dtype, scheme, d, dp, T, bits, group);
  float* Dh = one_pass ? reinterpret_cast<float*>(ws_at(ws, L.D_sqrt)) : nullptr;
  ttq_status st = run_statistic(X, dtype, d, T, p, lambda, alpha, L, ws, D, Dr, xh, xb, s, Dh);
  if (st != TTQ_OK || dp == 0) return st;
  if (one_pass) {
    // (2)-(3) at a few tokens: W read once, quantised and multiplied in one
    // kernel; no codes are written
    return run_single_pass(W, Dh, xh, X, A, B, d, dp, T, r, bits, group, nullptr, nullptr,
                           nullptr, Y, y_dtype == TTQ_F32, ws, L, s, true);
  }

  // (2) codes, scales, zeros of Q[W D^{1/2}]
  uint32_t* codes = reinterpret_cast<uint32_t*>(ws_at(ws, L.codes));
  uint16_t* scales = reinterpret_cast<uint16_t*>(ws_at(ws, L.scales));
  uint16_t* zeros = reinterpret_cast<uint16_t*>(ws_at(ws, L.zeros));
  void* wq = materialize_w(dp, T, bits, d) ? ws_at(ws, L.wq) : nullptr;
  // with the materialised weight the product reads W_hat alone: the codes,
  // scales and zeros are not written
  uint32_t* codes_out = wq ? nullptr : codes;
  uint16_t* scales_out = wq ? nullptr : scales;
  uint16_t* zeros_out = wq ? nullptr : zeros;
  st = cuda_status(scheme == TTQ_QSCHEME_FP8_E4M3
                       ? launch_qdq_fp8(W, f32, dp, d, D, group, codes_out, scales_out, zeros_out,
                                        status, device_sms(), s, true, wq)
                       : launch_qdq_pack(W, f32, dp, d, D, bits, group, codes_out, scales_out,
                                         zeros_out, status, device_sms(), s, true, wq,
                                         scheme == TTQ_QSCHEME_SYMMETRIC));
  if (st != TTQ_OK || T == 0) return st;

  // (3) Y = W_hat X (+ B (A X))
  const void* Ab = A;
  const void* Bb = B;
  if (f32 && r > 0) {
    void* ab = ws_at(ws, L.ab);
    void* bb = static_cast<uint8_t*>(ab) + static_cast<size_t>(r) * d * 2;
    st = cuda_status(launch_to_bf16(static_cast<const float*>(A), ab, r * d, s));
    if (st == TTQ_OK) st = cuda_status(launch_to_bf16(static_cast<const float*>(B), bb, dp * r, s));
    if (st != TTQ_OK) return st;
    Ab = ab;
    Bb = bb;
  }
  float* ypart = wq && L.ypart != 0 ? reinterpret_cast<float*>(ws_at(ws, L.ypart)) : nullptr;
  return run_gemm(codes, scales, zeros, xh, f32 ? xb : X, Ab, Bb, d, dp, T, r, bits, group, Y,
                  y_dtype == TTQ_F32, ws, L, s, true, wq, ypart);
}

ttq_status ttq_linear_forward(const void* X, const void* W, const void* A, const void* B,
                              ttq_dtype dtype, int64_t d, int64_t dp, int64_t T, int64_t r,
                              float p, float lambda, float alpha, int bits, int group, void* Y,
                              ttq_dtype y_dtype, void* ws, size_t ws_bytes, void* stream) {
  return ttq_linear_forward_ex(X, W, A, B, dtype, d, dp, T, r, p, lambda, alpha, bits, group,
                               TTQ_QSCHEME_ASYMMETRIC, Y, y_dtype, ws, ws_bytes, stream);
}

size_t ttq_lowrank_workspace_size(int64_t dp, int64_t d, int64_t r, int64_t oversample) {
  if (dp < 1 || d < 1 || r < 1 || oversample < 0 || r + oversample > 96) return 0;
  return ttq::lowrank_layout(dp, d, r + oversample).total;
}

ttq_status ttq_lowrank_init(const void* W, ttq_dtype dtype, int64_t dp, int64_t d, int64_t r,
                            int64_t oversample, int power_iters, const float* Omega, void* B,
                            void* A, void* W_res, void* ws, size_t ws_bytes, void* stream) {
  if (dtype != TTQ_F32 && dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (dp < 1 || d < 1 || r < 1 || oversample < 0 || power_iters < 0 || power_iters > 16)
    return TTQ_ERR_INVALID_ARG;
  const int64_t l = r + oversample;
  if (l > 96 || l > dp || l > d) return TTQ_ERR_UNSUPPORTED;
  if (dp > (int64_t{1} << 31) || d > (int64_t{1} << 31)) return TTQ_ERR_UNSUPPORTED;
  if (W == nullptr || Omega == nullptr || B == nullptr || A == nullptr) return TTQ_ERR_INVALID_ARG;
  const void* ptrs[] = {W, Omega, B, A, W_res};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTQ_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTQ_ERR_INVALID_ARG;
  if (ws_bytes < ttq::lowrank_layout(dp, d, l).total) return TTQ_ERR_WORKSPACE;
  return cuda_status(ttq::launch_lowrank_init(W, dtype == TTQ_BF16, dp, d, r, l, power_iters, Omega,
                                              B, A, W_res, ws, device_sms(),
                                              static_cast<cudaStream_t>(stream)));
}

ttq_status ttq_get_status(const void* ws, uint32_t* flags) {
  if (ws == nullptr) return TTQ_ERR_INVALID_ARG;
  uint32_t f = 0;
  if (cudaMemcpy(&f, ws, sizeof(f), cudaMemcpyDeviceToHost) != cudaSuccess) return TTQ_ERR_CUDA;
  if (flags) *flags = f;
  return ttq_status_from_flags(f);
}

ttq_status ttq_status_from_flags(uint32_t flags) {
  if (flags & TTQ_FLAG_TIMEOUT) return TTQ_ERR_TIMEOUT;
  if (flags & ~TTQ_FLAG_RANK_DEFICIENT) return TTQ_ERR_NONFINITE;
  return TTQ_OK;
}

const char* ttq_status_string(ttq_status s) {
  switch (s) {
    case TTQ_OK: return "ok";
    case TTQ_ERR_INVALID_ARG: return "invalid argument";
    case TTQ_ERR_UNSUPPORTED: return "unsupported parameter combination";
    case TTQ_ERR_CUDA: return "CUDA error";
    case TTQ_ERR_NONFINITE: return "non-finite value or binary16 scale overflow";
    case TTQ_ERR_TIMEOUT: return "device pipeline wait timed out";
    case TTQ_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* ttq_version(void) { return "0.2.0"; }

}  // extern "C"
