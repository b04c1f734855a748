// Host-side launchers of the TTQ kernels (internal to libttq.so).  Each
// returns cudaSuccess or the launch error; argument checking is done by the
// C ABI layer (ttq_api.cu) before these are called.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace ttq {

// Launches `kernel`; with pdl the launch may overlap the previous kernel on
// the stream (programmatic dependent launch: the kernel waits on the device
// before it reads that kernel's outputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Number of token splits of the statistic pass and the rows each covers.
void act_norm_plan(int64_t d, int64_t T, int num_sms, int64_t* splits, int64_t* rows_per_split);

// Step (1): D, D^{-1/2} from X [T][d].  `partial` holds splits x d doubles,
// `counters` ceil(d/256) uint32 that start (and are left) at zero.  When
// xh is non-null X is also written out as binary16 [T][d] (flag X_RANGE if
// some |x| > 65504); when xb is non-null a float32 X is also written out as
// bf16 [T][d].  When Dh is non-null it also receives sqrtf(D) (binary32,
// correctly rounded: the quantiser's h).
cudaError_t launch_act_norm(const void* X, bool x_f32, int64_t d, int64_t T, float p,
                            float lambda, float alpha, int64_t splits, int64_t rows_per_split,
                            double* partial, uint32_t* counters, float* D, float* Dr, void* xh,
                            void* xb, uint32_t* status, cudaStream_t stream, bool pdl = false,
                            float* Dh = nullptr);

// h = sqrtf(D) (binary32, correctly rounded) for d channels.
cudaError_t launch_sqrt_f32(const float* D, float* h, int64_t d, cudaStream_t stream);

// Whether launch_act_norm_scale would run (on the current device).
bool act_norm_scale_fused(bool x_f32, int64_t splits, int64_t rows_per_split, float p);

// Step (1) fused with the binary16 operand X D^(-1/2) (written to xh, which
// must be non-null; xb as for launch_act_norm).  One launch over the same
// splits as launch_act_norm, with D bit-identical to it; the splits of a
// 128-channel column block are one thread-block cluster.  X is read once and
// held in registers.  Launches only when each thread's rows of X fit in its
// registers (rows_per_split <= 256 for bf16, 128 for float32), there are at
// most 8 splits and such a cluster can be resident; *launched tells whether
// it ran (when it did not, nothing was queued and the result is
// cudaSuccess).
cudaError_t launch_act_norm_scale(const void* X, bool x_f32, int64_t d, int64_t T, float p,
                                  float lambda, float alpha, int64_t splits,
                                  int64_t rows_per_split, float* D, float* Dr, void* xh, void* xb,
                                  uint32_t* status, cudaStream_t stream, bool* launched,
                                  float* Dh = nullptr);

// Tensor map of a bf16 matrix [rows][cols] (row stride cols elements, a
// multiple of 8; base 16-byte aligned), loaded as box_rows x box_cols tiles
// (each at most 256) without swizzle: row-major in shared memory, rows past
// the matrix zero-filled.  False when the driver or the sizes do not allow it.
bool encode_bf16_box(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int box_cols,
                     int box_rows);

// Step (2): codes, scales, zeros of Q[W D^{1/2}] (D may be null); with wq
// non-null also the dequantised weight s (q - z) as binary16 [dp][d].
// symmetric: the symmetric quantiser (zero point 2^(b-1)).
cudaError_t launch_qdq_pack(const void* W, bool w_f32, int64_t dp, int64_t d, const float* D,
                            int bits, int group, uint32_t* codes, uint16_t* scales,
                            uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream, bool pdl = false, void* wq = nullptr,
                            bool symmetric = false);

// float32 -> bf16 copy of n elements (n % 8 == 0).
cudaError_t launch_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream);

// X' [T][d] = binary16(X[t][i] * Dr[i]) from float32, bf16 or binary16 X
// (Dr null: plain conversion); d % 8 == 0; flags X_RANGE if some
// |X'| > 65504.
constexpr int kSrcF32 = 0;
constexpr int kSrcBF16 = 1;
constexpr int kSrcF16 = 2;
cudaError_t launch_scale_to_f16(const void* src, int src_kind, const float* Dr, void* dst,
                                int64_t T, int64_t d, uint32_t* status, int num_sms,
                                cudaStream_t stream, bool pdl = false);

// Steps (2)-(3) on the tensor cores.
struct GemmArgs {
  // dequantised A operand (bits != 0) ...
  const uint32_t* codes = nullptr;
  const uint16_t* scales = nullptr;
  const uint16_t* zeros = nullptr;
  int bits = 0;               // 0: A operand loaded by TMA from tmA0 (plain mode)
  int group = 0;
  // sizes
  int64_t K = 0;        // reduction length of the main part (d)
  int64_t M = 0;        // output rows (d', or r for the A X product)
  int64_t T = 0;        // tokens
  int64_t K_tail = 0;   // low-rank reduction length r (0: none)
  // output Y[t][j] at Y + t * ldy + j
  void* Y = nullptr;
  int64_t ldy = 0;
  bool y_f32 = false;
  uint32_t* status = nullptr;
  bool a_f16 = false;      // plain mode: the A operand (maps.a0) is binary16, not bf16
  bool codes_tma = false;  // codes tile loaded by TMA (maps.c0); else per-thread loads
  bool y_tma = false;      // bf16 Y stored by TMA (maps.y, box block_m x block_n)
  // split-K (plain mode only): split z of k_splits covers K blocks
  // [z * kb_per_split, (z + 1) * kb_per_split), the last one the rest of the
  // main blocks and the low-rank tail, and writes its float32 partial
  // product to Y + z * split_stride (y_f32 must be set)
  int k_splits = 1;
  int kb_per_split = 0;
  int64_t split_stride = 0;
};

struct GemmMaps {
  CUtensorMap a0;  // plain A operand [M][K] bf16 or binary16 (bits == 0), box 64 x block_m
  CUtensorMap b0;  // binary16 X D^(-1/2) [T][K] with codes (bits != 0); bf16 X in the plain mode
  CUtensorMap a1;  // low-rank B [M][r] bf16
  CUtensorMap b1;  // A X [T][r] bf16
  CUtensorMap c0;  // packed codes [M][K*bits/32] uint32, box gemm_code_tile_words x block_m
  CUtensorMap y;   // bf16 Y [T][ldy], box 32 x 16 (rows of W x tokens), no swizzle
};

// Steps (2)-(3) for T <= 16 tokens: Y[t][j] = sum_i s (q - z) Xh[t][i]
// (+ sum_k Blr[j][k] AX[t][k] when r > 0, both bf16) with the codes
// dequantised in registers for warp-level tensor-core MMAs.  K a multiple
// of 64 (128 for INT3), group a power of two >= 32; Y [T][ldy] float32 or
// bf16.
struct DecodeArgs {
  const uint16_t* scales = nullptr;  // [M][K / group] binary16
  const uint16_t* zeros = nullptr;
  int64_t K = 0, M = 0, T = 0;
  int bits = 4, group = 128;
  const void* Blr = nullptr;         // bf16 [M][r]
  const void* AX = nullptr;          // bf16 [T][ax_ld]
  int64_t r = 0, ax_ld = 0;
  void* Y = nullptr;
  int64_t ldy = 0;
  bool y_f32 = false;
  uint32_t* status = nullptr;
};
// The 3-D tensor maps it reads.  tmC: the codes as uint32 seen as
// [K bits / 32 / piece_words][M][piece_words] (piece stride piece_words
// words, row stride K bits / 32 words), box piece_words x code_rows x
// code_pieces, no swizzle.  tmX: binary16 Xh seen as [K / unit_k][T][unit_k]
// (unit stride unit_k, token stride K), box unit_k x x_tokens x x_units,
// 128-byte swizzle.
struct DecodeMapShape {
  int piece_words, code_rows, code_pieces, unit_k, x_tokens, x_units;
};
DecodeMapShape decode_map_shape(int bits, int T);
cudaError_t launch_decode_gemm(const DecodeArgs& a, const CUtensorMap& tmC,
                               const CUtensorMap& tmX, cudaStream_t stream, bool pdl = false);

// Steps (2)-(3) in one pass over W for T <= 16 tokens: quantise bf16 W
// [M][K] with sqrt(D) (Dh), multiply by binary16 X' [T][K] (tmX) on
// warp-level MMAs, add B (A X) (bf16, when r > 0) and store Y [T][ldy];
// codes, scales and zeros (all three or none) are stored as the quantiser
// stores them.  K a multiple of 128, group 32, 64 or 128, bits 2..4.
// Persistent grid of fused_decode_plan().grid CTAs over row tiles of 256;
// `part` holds plan.part_floats floats, `tickets` plan.row_tiles uint32
// that are zero before and after the call.  tmW: bf16 W [M][K], box 64 x
// 256, 128-byte swizzle; tmX: binary16 X' [T][K], box 64 x (T <= 8 ? 8 :
// 16), 128-byte swizzle.
constexpr int kFusedDecodePlanSMs = 148;     // fixed so the layout is device-independent
constexpr int64_t kFusedDecodeMaxTiles = 4096;
struct FusedDecodePlan {
  int grid;
  int64_t row_tiles, units, part_floats;
};
FusedDecodePlan fused_decode_plan(int64_t dp, int64_t d, int64_t T);
int fused_decode_rows();   // rows of W per unit (the W box height)
bool fused_decode_supported(int64_t dp, int64_t d, int64_t T, int bits, int group);
struct FusedDecodeArgs {
  const float* Dh = nullptr;
  int64_t K = 0, M = 0, T = 0;
  int bits = 4, group = 128;
  const void* Blr = nullptr;   // bf16 [M][r]
  const void* AX = nullptr;    // bf16 [T][ax_ld]
  int64_t r = 0, ax_ld = 0;
  void* Y = nullptr;
  int64_t ldy = 0;
  bool y_f32 = false;
  uint32_t* codes = nullptr;
  uint16_t* scales = nullptr;
  uint16_t* zeros = nullptr;
  float* part = nullptr;
  uint32_t* tickets = nullptr;
  uint32_t* status = nullptr;
};
cudaError_t launch_fused_decode(const FusedDecodeArgs& a, const CUtensorMap& tmW,
                                const CUtensorMap& tmX, cudaStream_t stream, bool pdl = false);

// Step (2) with FP8 (E4M3) codes: one byte per weight (4 per word), the
// symmetric per-group scale binary16 round-up(max|x| / 448), zeros +0;
// with wq also the binary16 s * e4m3(code).
cudaError_t launch_qdq_fp8(const void* W, bool w_f32, int64_t dp, int64_t d, const float* D,
                           int group, uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                           uint32_t* status, int num_sms, cudaStream_t stream, bool pdl, void* wq);

// Static low-rank initialisation (B, A from a randomised truncated SVD of
// W; residual W - B A).  Workspace offsets (bytes) past the 4 KiB status
// header; l = r + oversample.
struct LowrankLayout {
  size_t Y, Q, Bt, partial, G, Rinv, U, sigma, inv_sigma, total;
  int64_t partial_floats;
};
LowrankLayout lowrank_layout(int64_t dp, int64_t d, int64_t l);
size_t lowrank_small_smem(int l, bool eig);
cudaError_t launch_lowrank_init(const void* W, bool w_bf16, int64_t dp, int64_t d, int64_t r, int64_t l,
                                int power_iters, const float* Omega, void* Bout, void* Aout, void* Wres,
                                void* ws, int num_sms, cudaStream_t stream);

// Split-K plan of the low-rank product A X (M = r rows of A, T tokens, K =
// d): the number of K splits that brings its few output tiles up to about
// one wave on num_sms SMs with at least 4 K blocks of 64 per split (1: no
// split), and the K blocks each split covers.
struct AxSplit {
  int splits, kb_per_split;
};
AxSplit ax_split_plan(int64_t r, int64_t T, int64_t d, int num_sms);

// The low-rank A X product for 17 to kAxMaxTokens tokens on warp-level
// MMAs: plan.splits slices of plan.kb_per_split channels of the reduction
// (512 for r <= 32, else 256), one CTA per 64 tokens and slice.  With one
// slice it writes bf16 AX [T][ax_ld] itself; with more it writes the fp32
// partial sums P [splits][T][r] for launch_ax_reduce.  ax_mma_plan returns
// splits = 0 where it does not apply (other token counts, or r not a
// multiple of 8 in 8..96).
constexpr int64_t kAxMaxTokens = 512;
struct AxMmaPlan {
  int splits;   // channel slices (0: the kernel does not apply)
  int kc;       // channels per slice
};
AxMmaPlan ax_mma_plan(int64_t r, int64_t T, int64_t d);
cudaError_t launch_ax_mma(const void* A, const void* X, int64_t d, int64_t T, int64_t r,
                          const AxMmaPlan& plan, float* P, void* AX, int64_t ax_ld,
                          cudaStream_t stream, bool pdl);

// AX [T][ax_ld] bf16 = the sum over the splits, in split order, of the
// float32 partials P [splits][T][r] (one rounding at the end).
cudaError_t launch_ax_reduce(const float* P, int splits, int64_t T, int64_t r, void* AX,
                             int64_t ax_ld, cudaStream_t stream, bool pdl);

// Words per row of the code tile one K block of 64 channels needs.
int gemm_code_tile_words(int bits);

// Tile width along the tokens for T tokens.
int gemm_block_n(int64_t T);

// Tile shape of the product for this problem: block_m 128 or 256 rows of W
// (256 only with codes), block_n a multiple of 16 up to 256 tokens, chosen
// so that the CTAs fill the SMs in as few, as full waves as possible.
void gemm_tile_shape(int bits, int64_t M, int64_t T, int num_sms, int* block_m, int* block_n);

// Tile shape and K split of the product on the materialised binary16 weight
// (plain mode: M rows of W_hat, T tokens, K channels, K_tail low-rank
// channels): BM x BN tiles and `splits` parts of kb_per_split K blocks of 64
// (splits 1, kb_per_split 0: unsplit; the last part also takes the rest of
// the blocks and the low-rank tail).  Unsplit, the shape is gemm_tile_shape's;
// a split is taken where a time model that counts the tensor-core time, the
// operand traffic from L2 and the float32 partial sums with their reduction
// (launch_y_reduce) puts it well ahead.
struct GemmPlan {
  int block_m, block_n, splits, kb_per_split;
};
GemmPlan gemm_plan_plain(int64_t M, int64_t T, int64_t K, int64_t K_tail, int num_sms,
                         bool allow_split);

// Y (n elements, bf16 or float32) = the sum over the splits, in split order,
// of the float32 partials P [splits][n], rounded once.
cudaError_t launch_y_reduce(const float* P, int splits, int64_t n, void* Y, bool y_f32,
                            cudaStream_t stream, bool pdl);

// The operand boxes: a0/a1 are loaded as block_m x 64, b0/b1 as block_n x 64.
cudaError_t launch_dequant_gemm(const GemmArgs& args, const GemmMaps& maps, int block_n,
                                int block_m, cudaStream_t stream, bool pdl = false);

}  // namespace ttq
