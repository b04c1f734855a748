// Steps (2)-(3) of the TTQ layer for a few tokens (T <= 16):
//   Y[t][j] = sum_i s_jk (q_ji - z_jk) X'[t][i]  (+ sum_k B[j][k] AX[t][k])
// with X' = X D^(-1/2) in binary16 (gist.science/zh/paper/2603.19296,
// section 2.1 for W_hat, 2.2 for the static low-rank pair).
//
// With so few tokens the product is a matrix-vector product over the packed
// codes, and turning codes into tensor-core operands costs as much as
// reading them, so the kernel is laid out to spend few instructions per
// code.  One producer warp streams, per stage of 512 input channels, the
// code tile of the CTA's 64 rows of W and the matching 512 channels of X'
// into shared memory, one 3-D TMA copy each (few, large stages: issuing a
// stage costs the producer about as much as a consumer spends on a small
// one).  The code tile lands unit-major -- 64-channel units, each a block of
// 64 rows -- so the rows a warp reads at once sit 16 to 48 bytes apart, free
// of bank conflicts.  Eight consumer warps -- two groups of 32 rows x four
// quarters of every stage (units 2kq, 2kq + 1) -- turn the codes into
// binary16 operands in registers and run warp-level MMAs (m16n8k16,
// binary16 x binary16 -> fp32); each warp's two 16-row tiles share the X'
// operand.  The quarters are added in a fixed order at the end, so the
// result is deterministic.
//
// The order of the 16 products inside one MMA is free as long as the A and
// B operands agree on it.  Each lane (g = lane / 4, c = lane % 4) owns
// channels 16c .. 16c + 15 of each 64-channel half ("unit") of a stage and
// pairs codes the way the packing makes cheap: a code at bit b of a 16-bit
// half, OR-ed into the exponent of m = 2^(10 - b), reads as the binary16
// m + q, so INT4 channels (i, i + 4) and INT2 (i, i + 8) of a unit come out
// of a word with one mask each (INT3: (2i, 2i + 1) after a shift).  The
// matching pairs of X' are put together with byte permutes.  The X' tiles
// are 128-byte swizzled, which makes their reads free of bank conflicts.
//
// The operand is (m + q) - (m + z) = q - z, exact in binary16; FP8 (E4M3)
// codes (one byte per channel) convert to their binary16 values exactly and
// need no zero point (the blog.lo0.es comparison with FP8: the activation-
// aware scale feeding an FP8 code).  For up to 8
// tokens with quantisation groups that span whole stages (group >= 128) s
// multiplies the fp32 sum of a stage once per row; otherwise the operand is
// the binary16 s (q - z) (one rounding), as in the large-tile product.
//
// Register layout of m16n8k16 (PTX ISA, warp-level MMA): the A registers
// hold rows g and g + 8 at the lane's K pair 0 (registers 0, 1) and K pair 1
// (registers 2, 3); B holds the same two K pairs of column (token) g; C
// holds rows g, g + 8 at columns 2c, 2c + 1.
//
// Every barrier wait is bounded (1 s); a wait that gives up sets
// TTQ_FLAG_TIMEOUT, stops the CTA's other warps, lets the copies in flight
// land, and the CTA returns without storing Y.

#include <cuda_fp8.h>

#include <atomic>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kRowGroups = 2;                   // 32-row groups per CTA
constexpr int kRowsPerCta = 32 * kRowGroups;
constexpr int kQuarters = 4;                    // consumer warps per row group
constexpr int kConsumers = kRowGroups * kQuarters;
constexpr int kUnitK = 64;                      // channels per unit
constexpr int kUnits = 8;                       // units per stage
constexpr int kStageK = kUnitK * kUnits;

// The code tile is copied in pieces of one unit (two for INT3, whose unit
// of 24 bytes is not a multiple of 16): [piece][row][piece bytes].
template <int BITS>
constexpr int piece_units() { return BITS == 3 ? 2 : 1; }
template <int BITS>
constexpr int piece_words() { return kUnitK * BITS / 32 * piece_units<BITS>(); }
template <int BITS>
constexpr int pieces() { return kUnits / piece_units<BITS>(); }
template <int BITS>
constexpr uint32_t code_tile_bytes() { return kRowsPerCta * kStageK * BITS / 8; }
// X' of a stage: [unit][8 NTT tokens][64 channels], 128-byte swizzled
template <int NTT>
constexpr uint32_t xh_tile_bytes() { return kUnits * 8u * NTT * 128u; }
template <int BITS, int NTT>
constexpr int num_stages() { return BITS == 8 ? 2 : (NTT == 1 ? 4 : 3); }
template <int BITS, int NTT>
constexpr uint32_t stage_bytes() {
  return (xh_tile_bytes<NTT>() + code_tile_bytes<BITS>() + 1023u) & ~1023u;
}
template <int BITS, int NTT>
constexpr size_t decode_smem_bytes() {
  return static_cast<size_t>(num_stages<BITS, NTT>()) * stage_bytes<BITS, NTT>() + 1024;
}

__device__ __forceinline__ void mma_m16n8k16_f16(float (&c)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  __half2 v;
  memcpy(&v, &u, 4);
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Number of distinct magics m a unit's pairs use, and pair p's index into
// them: INT4 {1024, 64}; INT2 {1024, 256, 64, 16, 4}; INT3 {1024}.
template <int BITS>
constexpr int num_kinds() { return BITS == 4 ? 2 : (BITS == 2 ? 5 : 1); }
template <int BITS>
__device__ __forceinline__ constexpr int pair_kind(int p) {
  return BITS == 4 ? (p & 1) : (BITS == 2 ? (p < 5 ? p : p - 5) : 0);
}
template <int BITS>
__device__ __forceinline__ constexpr uint32_t kind_magic(int k) {
  return BITS == 2 ? (k == 0 ? 0x6400u : k == 1 ? 0x5C00u : k == 2 ? 0x5400u
                                       : k == 3 ? 0x4C00u : 0x4400u)
                   : (k == 0 ? 0x6400u : 0x5400u);
}

// Two E4M3 codes (low 16 bits of v) as a binary16 pair: exact, every E4M3
// value is a binary16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// (m + q) pairs P[0..7] of the lane's 16 channels of unit u of its piece,
// for one row (row_addr: the row's first byte in the piece).  INT4: P[i] =
// channels (i, i + 4), P[4 + i] = (8 + i, 12 + i); INT2: P[i] = (i, i + 8);
// INT3: P[i] = (2i, 2i + 1); 8-bit E4M3 codes: the binary16 values of
// channels (2i, 2i + 1) themselves (zero point 0).

template <int BITS>
__device__ __forceinline__ void code_pairs(uint32_t row_addr, int u, int c, uint32_t (&P)[8]) {
  if (BITS == 8) {
    // E4M3 codes, one byte per channel in channel order: the lane's 16
    // channels are 16 bytes, and each byte pair converts to the binary16
    // pair (2i, 2i + 1) exactly (every E4M3 value is a binary16 value)
    const uint4 w = lds128(row_addr + 64 * u + 16 * c);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      P[2 * k] = e4m3x2_to_h2(ws[k]);
      P[2 * k + 1] = e4m3x2_to_h2(ws[k] >> 16);
    }
  } else if (BITS == 4) {
    const uint2 w = lds64(row_addr + 32 * u + 8 * c);
    const uint32_t lo8 = w.x >> 8, hi8 = w.y >> 8;
    P[0] = (w.x & 0x000F000Fu) | 0x64006400u;   // channels 0, 4
    P[1] = (w.x & 0x00F000F0u) | 0x54005400u;   // 1, 5
    P[2] = (lo8 & 0x000F000Fu) | 0x64006400u;   // 2, 6
    P[3] = (lo8 & 0x00F000F0u) | 0x54005400u;   // 3, 7
    P[4] = (w.y & 0x000F000Fu) | 0x64006400u;
    P[5] = (w.y & 0x00F000F0u) | 0x54005400u;
    P[6] = (hi8 & 0x000F000Fu) | 0x64006400u;
    P[7] = (hi8 & 0x00F000F0u) | 0x54005400u;
  } else if (BITS == 2) {
    const uint32_t w = lds32(row_addr + 16 * u + 4 * c);
    const uint32_t w10 = w >> 10;
    P[0] = (w & 0x00030003u) | 0x64006400u;     // channels 0, 8
    P[1] = (w & 0x000C000Cu) | 0x5C005C00u;     // 1, 9
    P[2] = (w & 0x00300030u) | 0x54005400u;     // 2, 10
    P[3] = (w & 0x00C000C0u) | 0x4C004C00u;     // 3, 11
    P[4] = (w & 0x03000300u) | 0x44004400u;     // 4, 12
    P[5] = (w10 & 0x00030003u) | 0x64006400u;   // 5, 13
    P[6] = (w10 & 0x000C000Cu) | 0x5C005C00u;   // 6, 14
    P[7] = (w10 & 0x00300030u) | 0x54005400u;   // 7, 15
  } else {
    // the unit's channels 16c.. start at bit 48c of the unit's 192 bits:
    // word 6u + (3c >> 1), plus 16 bits for odd c
    const uint32_t wi = 6u * u + (static_cast<uint32_t>(3 * c) >> 1);
    const uint64_t win = static_cast<uint64_t>(lds32(row_addr + 4 * wi)) |
                         (static_cast<uint64_t>(lds32(row_addr + 4 * wi + 4)) << 32);
    const uint64_t b = win >> ((c & 1) * 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t t = static_cast<uint32_t>(b >> (6 * i));
      P[i] = (t & 0x7u) | ((t & 0x38u) << 13) | 0x64006400u;
    }
  }
}

// The X' pairs B[0..7] matching code_pairs, from the unit's 16 channels
// X[m] = channels (2m, 2m + 1).
template <int BITS>
__device__ __forceinline__ void x_pairs(const uint32_t (&X)[8], uint32_t (&B)[8]) {
  if (BITS == 4) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
      B[i] = __byte_perm(X[i >> 1], X[2 + (i >> 1)], sel);
      B[4 + i] = __byte_perm(X[4 + (i >> 1)], X[6 + (i >> 1)], sel);
    }
  } else if (BITS == 2) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      B[i] = __byte_perm(X[i >> 1], X[4 + (i >> 1)], (i & 1) ? 0x7632u : 0x5410u);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) B[i] = X[i];
  }
}

// PS: s applied per 128-channel block to fp32 sums of exact (q - z)
// operands (group >= 128); otherwise binary16 s (q - z) operands.
template <int BITS, int NTT, bool PS>
__global__ void __launch_bounds__(32 * (1 + kConsumers), 2) ttq_decode_kernel(
    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
    const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros, int K, int M,
    int T, int group_shift, const __nv_bfloat16* __restrict__ Blr,
    const __nv_bfloat16* __restrict__ AX, int r, int ax_ld, void* __restrict__ Y, int ldy,
    int y_f32, uint32_t* status) {
  constexpr int kStages = num_stages<BITS, NTT>();
  extern __shared__ uint8_t dsm[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ int abort_s;
  __shared__ float red[kQuarters - 1][kRowGroups][2][NTT][4][32];   // quarters 1..3
  constexpr uint32_t kXh = xh_tile_bytes<NTT>();
  constexpr uint32_t kCode = code_tile_bytes<BITS>();
  constexpr uint32_t kStage = stage_bytes<BITS, NTT>();
  constexpr uint32_t kPieceRow = piece_words<BITS>() * 4;        // bytes of a row in a piece
  constexpr uint32_t kPiece = kPieceRow * kRowsPerCta;
  constexpr int kKinds = num_kinds<BITS>();
  constexpr int kUnitsSz = PS ? 1 : 2;           // (s, z) per row: per block or per unit
  const uint32_t smem = (smem_addr(dsm) + 1023u) & ~1023u;
  uint8_t* smem_ptr = dsm + (smem - smem_addr(dsm));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nsteps = (K + kStageK - 1) / kStageK;
  const int row0 = blockIdx.x * kRowsPerCta;
  volatile int* abort_flag = &abort_s;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    abort_s = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmC);
    prefetch_tensormap(&tmX);
  }
  __syncthreads();
  allow_dependents_launch();
  grid_dependency_wait();

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int st = 0; st < nsteps; ++st) {
        const int s = st % kStages;
        const uint32_t ph = static_cast<uint32_t>(st / kStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          *abort_flag = 1;
          set_flag(status, TTQ_FLAG_TIMEOUT);
          break;
        }
        uint8_t* base = smem_ptr + s * kStage;
        mbar_arrive_expect_tx(&full[s], kXh + kCode);
        tma_load_3d(&tmX, &full[s], base, 0, 0, st * kUnits);
        tma_load_3d(&tmC, &full[s], base + kXh, 0, row0, st * pieces<BITS>());
        issued = st + 1;
      }
      if (*abort_flag) {
        // the copies in flight land before the CTA's shared memory goes away
        int never = 0;
        for (int st = issued > kStages ? issued - kStages : 0; st < issued; ++st)
          mbar_wait(&full[st % kStages], static_cast<uint32_t>(st / kStages) & 1u, &never);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  // warp 1 + rg + 2 kq: rows 32 rg + {g, g + 8, g + 16, g + 24} of the CTA
  // (two 16-row MMA tiles), units 2 kq and 2 kq + 1 of every stage
  const int cw = warp - 1;
  const int rg = cw % kRowGroups;
  const int kq = cw / kRowGroups;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int ngroups = K >> group_shift;
  int rloc[4];
  const uint16_t* srow[4];
  const uint16_t* zrow[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    rloc[i] = 32 * rg + g + 8 * i;
    const int row = row0 + rloc[i] < M ? row0 + rloc[i] : M - 1;
    srow[i] = scales + static_cast<int64_t>(row) * ngroups;
    zrow[i] = zeros + static_cast<int64_t>(row) * ngroups;
  }
  // s | z << 16 of the lane's four rows for stage st and unit 2 kq + v (the
  // lane's 16 channels lie in one quantisation group; with PS the whole
  // 128-channel block does); past K the group index is clamped (the
  // matching X' is zero)
  auto load_sz = [&](int st, int v, uint32_t (&dst)[4]) {
    int gi = (st * kStageK + (2 * kq + v) * kUnitK + (PS ? 0 : 16 * c)) >> group_shift;
    gi = gi < ngroups ? gi : ngroups - 1;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = static_cast<uint32_t>(__ldg(srow[i] + gi)) |
               (static_cast<uint32_t>(__ldg(zrow[i] + gi)) << 16);
  };
  // (s, z) run one stage ahead, in two slots whose index is static after
  // unrolling (moving a register still being loaded would wait for the load)
  uint32_t sz[2][kUnitsSz][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int v = 0; v < kUnitsSz; ++v) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sz[j][v][i] = 0u;
      if (j < nsteps) load_sz(j, v, sz[j][v]);
    }
  // with one token tile the two units accumulate apart (four independent
  // MMA chains per warp instead of two); added in unit order
  constexpr int kUA = NTT == 1 ? 2 : 1;
  float acc[kUA][2][NTT][4];
#pragma unroll
  for (int ua = 0; ua < kUA; ++ua)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt)
        acc[ua][mt][tt][0] = acc[ua][mt][tt][1] = acc[ua][mt][tt][2] = acc[ua][mt][tt][3] = 0.f;
  bool ok = true;

  for (int i0 = 0; i0 < nsteps && ok; i0 += 2) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int st = i0 + j;
      if (st >= nsteps) break;
      const int s = st % kStages;
      const uint32_t ph = static_cast<uint32_t>(st / kStages) & 1u;
      if (!mbar_wait(&full[s], ph, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          set_flag(status, TTQ_FLAG_TIMEOUT);
        }
        ok = false;
        break;
      }
      const uint32_t base = smem + s * kStage;
      float part[kUA][2][NTT][4];
      if (PS) {
#pragma unroll
        for (int ua = 0; ua < kUA; ++ua)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int tt = 0; tt < NTT; ++tt)
              part[ua][mt][tt][0] = part[ua][mt][tt][1] = part[ua][mt][tt][2] = part[ua][mt][tt][3] = 0.f;
      }
      float sf[4];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int u = 2 * kq + v;                  // unit of the stage
        if (st * kStageK + u * kUnitK >= K) break;  // past the end of the row
        const int vs = PS ? 0 : v;
        // (m + z) pairs of the four rows for every magic m in use (exact),
        // and s (a binary16 pair, or a float for the per-block scaling)
        uint32_t zc[4][kKinds], s2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t zz = __byte_perm(sz[j][vs][i], 0u, 0x3232u);   // z in both halves
          const uint32_t ss = __byte_perm(sz[j][vs][i], 0u, 0x1010u);   // s in both halves
#pragma unroll
          for (int k = 0; k < kKinds; ++k)
            zc[i][k] = h2_bits(__hadd2(bits_h2(zz), bits_h2(kind_magic<BITS>(k) * 0x00010001u)));
          s2[i] = ss;
          if (PS && v == 0) sf[i] = __half2float(__ushort_as_half(static_cast<uint16_t>(ss & 0xFFFFu)));
        }
        const int piece = u / piece_units<BITS>();
        const int h = u % piece_units<BITS>();
        const uint32_t prow = base + kXh + static_cast<uint32_t>(piece) * kPiece +
                              static_cast<uint32_t>(32 * rg + g) * kPieceRow;
        uint32_t P[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          code_pairs<BITS>(prow + 8u * i * kPieceRow, h, c, P[i]);
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const __half2 x = BITS == 8 ? bits_h2(P[i][p])
                                        : __hsub2(bits_h2(P[i][p]), bits_h2(zc[i][pair_kind<BITS>(p)]));
            P[i][p] = PS ? h2_bits(x) : h2_bits(__hmul2(x, bits_h2(s2[i])));
          }
        }
        // the unit's 16 channels of X' are chunks 2c, 2c + 1 of the 128-byte
        // token rows of unit u, swizzled by row & 7 (= g)
        const uint32_t xrow = base + static_cast<uint32_t>(u) * (8u * NTT * 128u) +
                              static_cast<uint32_t>(g) * 128u;
        const uint32_t off0 = (static_cast<uint32_t>(2 * c) ^ static_cast<uint32_t>(g)) << 4;
        const uint32_t off1 = (static_cast<uint32_t>(2 * c + 1) ^ static_cast<uint32_t>(g)) << 4;
#pragma unroll
        for (int tt = 0; tt < NTT; ++tt) {
          const uint4 x0 = lds128(xrow + 1024u * tt + off0);
          const uint4 x1 = lds128(xrow + 1024u * tt + off1);
          const uint32_t X[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t B[8];
          x_pairs<BITS>(X, B);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              const uint32_t a[4] = {P[2 * mt][2 * k], P[2 * mt + 1][2 * k], P[2 * mt][2 * k + 1],
                                     P[2 * mt + 1][2 * k + 1]};
              const int ua = kUA > 1 ? v : 0;
              mma_m16n8k16_f16(PS ? part[ua][mt][tt] : acc[ua][mt][tt], a, B[2 * k], B[2 * k + 1]);
            }
          }
        }
      }
      // refill this slot with the (s, z) of the stage after next
      if (st + 2 < nsteps) {
#pragma unroll
        for (int v = 0; v < kUnitsSz; ++v) load_sz(st + 2, v, sz[j][v]);
      }
      if (PS && st * kStageK + 2 * kq * kUnitK < K) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int tt = 0; tt < NTT; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float x = part[0][mt][tt][e];
              if (kUA > 1) x += part[kUA - 1][mt][tt][e];
              acc[0][mt][tt][e] = fmaf(sf[2 * mt + (e >> 1)], x, acc[0][mt][tt][e]);
            }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // the low-rank term B (A X), bf16 operands in the plain register layout
  // (K pair 0 = k 2c, 2c + 1; K pair 1 = k 2c + 8, 2c + 9), on the last
  // quarter's warps
  if (kq == kQuarters - 1 && r > 0 && ok) {
    for (int k0 = 0; k0 < r; k0 += 16) {
      const int kc = k0 + 2 * c;
      const bool lo_ok = kc < r, hi_ok = kc + 8 < r;
      uint32_t a[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int rowa = row0 + rloc[2 * mt], rowb = row0 + rloc[2 * mt + 1];
        const __nv_bfloat16* ba = Blr + static_cast<int64_t>(rowa < M ? rowa : 0) * r;
        const __nv_bfloat16* bb = Blr + static_cast<int64_t>(rowb < M ? rowb : 0) * r;
        a[mt][0] = (rowa < M && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc)) : 0u;
        a[mt][1] = (rowb < M && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc)) : 0u;
        a[mt][2] = (rowa < M && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc + 8)) : 0u;
        a[mt][3] = (rowb < M && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc + 8)) : 0u;
      }
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt) {
        const int n = 8 * tt + g;
        const bool n_ok = n < T;
        const __nv_bfloat16* axn = AX + static_cast<int64_t>(n_ok ? n : 0) * ax_ld;
        const uint32_t b0 = (n_ok && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc)) : 0u;
        const uint32_t b1 = (n_ok && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc + 8)) : 0u;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) mma_m16n8k16_bf16(acc[0][mt][tt], a[mt], b0, b1);
      }
    }
  }

  // quarters 1..3 hand their sums to quarter 0 of the same rows, which adds
  // them in quarter order and stores Y: C rows g, g + 8 of tile mt are rows
  // rloc[2 mt], rloc[2 mt + 1]; columns 2c, 2c + 1 of token tile tt are
  // tokens 8 tt + 2c, 8 tt + 2c + 1
  if (!PS && kUA > 1) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][mt][tt][e] += acc[kUA - 1][mt][tt][e];
  }
  if (kq > 0) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[kq - 1][rg][mt][tt][e][lane] = acc[0][mt][tt][e];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
  if (kq > 0 || *abort_flag) return;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int tt = 0; tt < NTT; ++tt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = acc[0][mt][tt][e];
#pragma unroll
        for (int q = 0; q < kQuarters - 1; ++q) x += red[q][rg][mt][tt][e][lane];
        const int row = row0 + rloc[2 * mt + (e >> 1)];
        const int t = 8 * tt + 2 * c + (e & 1);
        if (row < M && t < T) {
          const int64_t at = static_cast<int64_t>(t) * ldy + row;
          if (y_f32) static_cast<float*>(Y)[at] = x;
          else static_cast<__nv_bfloat16*>(Y)[at] = __float2bfloat16_rn(x);
        }
      }
    }
  }
}

template <int BITS, int NTT, bool PS>
cudaError_t launch_decode_typed(const CUtensorMap& tmC, const CUtensorMap& tmX,
                                const DecodeArgs& a, int group_shift, cudaStream_t stream,
                                bool pdl) {
  constexpr size_t smem = decode_smem_bytes<BITS, NTT>();
  // the attribute belongs to a device: set once per device (the first
  // launch on it, normally outside any graph capture); host threads that
  // race here both set the same value
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t attr_err = cudaFuncSetAttribute(ttq_decode_kernel<BITS, NTT, PS>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(smem));
    if (attr_err != cudaSuccess) return attr_err;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_relaxed);
  }
  const dim3 grid(static_cast<unsigned>((a.M + kRowsPerCta - 1) / kRowsPerCta));
  return launch_kernel(ttq_decode_kernel<BITS, NTT, PS>, grid, dim3(32 * (1 + kConsumers)), smem,
                       stream, pdl, tmC, tmX, a.scales, a.zeros, static_cast<int>(a.K),
                       static_cast<int>(a.M), static_cast<int>(a.T), group_shift,
                       static_cast<const __nv_bfloat16*>(a.Blr),
                       static_cast<const __nv_bfloat16*>(a.AX), static_cast<int>(a.r),
                       static_cast<int>(a.ax_ld), a.Y, static_cast<int>(a.ldy), a.y_f32 ? 1 : 0,
                       a.status);
}

template <int BITS>
cudaError_t launch_decode_bits(const CUtensorMap& tmC, const CUtensorMap& tmX,
                               const DecodeArgs& a, int gs, cudaStream_t stream, bool pdl) {
  // two token tiles share each dequantised operand, and their block sums
  // would not fit in registers besides: s goes into the operand there
  if (a.T > 8) return launch_decode_typed<BITS, 2, false>(tmC, tmX, a, gs, stream, pdl);
  return a.group >= 2 * kUnitK
             ? launch_decode_typed<BITS, 1, true>(tmC, tmX, a, gs, stream, pdl)
             : launch_decode_typed<BITS, 1, false>(tmC, tmX, a, gs, stream, pdl);
}


// The low-rank A X product for 17 to 512 tokens, out[t][k] = sum_i
// A[k][i] X[t][i] (bf16 operands, fp32 sums): CTA (x, y) takes tokens
// 64 x .. 64 x + 63 and channels [y kc, (y + 1) kc) of the reduction, brings
// both operand slices into shared memory at once with asynchronous copies
// (zero-filled past T and d), and its four warps each multiply 16 tokens by
// all r rows of A with warp-level MMAs (m16n8k16, k ascending).  With one
// channel slice the CTA rounds its sums to bf16 AX [T][ax_ld]; otherwise it
// writes its fp32 partial sums to P [slice][T][r] for ax_reduce_kernel to add
// in slice order.  Rows of the shared tiles are padded by 16 bytes so that
// the fragment loads of a warp fall in 32 different banks.
constexpr int kAxTokens = 64;
constexpr int kAxThreads = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}

template <int NT>   // NT = r / 8 tiles of 8 rows of A
__global__ void __launch_bounds__(kAxThreads) ax_mma_kernel(
    const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ X, int64_t d, int64_t T,
    int kc, float* __restrict__ P, __nv_bfloat16* __restrict__ AX, int64_t ax_ld) {
  extern __shared__ __align__(16) __nv_bfloat16 ax_smem[];
  constexpr int R = 8 * NT;
  const int ld = kc + 8;                          // padded row, in elements
  __nv_bfloat16* sX = ax_smem;                    // [kAxTokens][ld]
  __nv_bfloat16* sA = ax_smem + kAxTokens * ld;   // [R][ld]
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kAxTokens;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * kc;
  allow_dependents_launch();
  grid_dependency_wait();   // X may come from the previous kernel

  // both slices, 16 bytes (8 channels) per copy; d % 8 == 0, so a chunk is
  // either inside d or wholly past it
  const int cpr = kc / 8;                         // chunks per row
  for (int c = threadIdx.x; c < (kAxTokens + R) * cpr; c += kAxThreads) {
    const int row = c / cpr, ch = c - row * cpr;
    const int64_t k = k0 + ch * 8;
    const bool in_x = row < kAxTokens;
    const int64_t grow = in_x ? t0 + row : row - kAxTokens;
    const bool valid = k < d && (!in_x || grow < T);
    const __nv_bfloat16* src = (in_x ? X : A) + (valid ? grow * d + k : 0);
    __nv_bfloat16* dst = (in_x ? sX + row * ld : sA + (row - kAxTokens) * ld) + ch * 8;
    cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(dst)), src, valid ? 16u : 0u);
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qr = lane >> 2, qc = (lane & 3) * 2;
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const __nv_bfloat16* xr0 = sX + (warp * 16 + qr) * ld + qc;
  const __nv_bfloat16* xr1 = xr0 + 8 * ld;
  const __nv_bfloat16* ar = sA + qr * ld + qc;
  const int ksteps = static_cast<int>(min(static_cast<int64_t>(kc), d - k0) + 15) / 16;
  for (int s = 0; s < ksteps; ++s) {
    const int kk = s * 16;
    uint32_t a[4];
    a[0] = *reinterpret_cast<const uint32_t*>(xr0 + kk);
    a[1] = *reinterpret_cast<const uint32_t*>(xr1 + kk);
    a[2] = *reinterpret_cast<const uint32_t*>(xr0 + kk + 8);
    a[3] = *reinterpret_cast<const uint32_t*>(xr1 + kk + 8);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const __nv_bfloat16* b = ar + j * 8 * ld + kk;
      mma_m16n8k16_bf16(acc[j], a, *reinterpret_cast<const uint32_t*>(b),
                        *reinterpret_cast<const uint32_t*>(b + 8));
    }
  }

  const bool partial = gridDim.y > 1;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t t = t0 + warp * 16 + qr + 8 * h;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int k = j * 8 + qc;
      if (partial) {
        float2* dst = reinterpret_cast<float2*>(P + (static_cast<int64_t>(blockIdx.y) * T + t) * R + k);
        *dst = make_float2(acc[j][2 * h], acc[j][2 * h + 1]);
      } else {
        *reinterpret_cast<__nv_bfloat162*>(AX + t * ax_ld + k) =
            __floats2bfloat162_rn(acc[j][2 * h], acc[j][2 * h + 1]);
      }
    }
  }
}

template <int NT>
cudaError_t launch_ax_mma_nt(const __nv_bfloat16* A, const __nv_bfloat16* X, int64_t d, int64_t T,
                             int kc, int splits, float* P, __nv_bfloat16* AX, int64_t ax_ld,
                             cudaStream_t stream, bool pdl) {
  const size_t smem = static_cast<size_t>(kAxTokens + 8 * NT) * (kc + 8) * 2;
  static std::atomic<size_t> attr_bytes[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || attr_bytes[dev].load(std::memory_order_relaxed) < smem) {
    const cudaError_t e = cudaFuncSetAttribute(ax_mma_kernel<NT>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_bytes[dev].store(smem, std::memory_order_relaxed);
  }
  const dim3 grid(static_cast<unsigned>((T + kAxTokens - 1) / kAxTokens), static_cast<unsigned>(splits));
  return launch_kernel(ax_mma_kernel<NT>, grid, dim3(kAxThreads), smem, stream, pdl, A, X, d, T, kc,
                       P, AX, ax_ld);
}

}  // namespace

DecodeMapShape decode_map_shape(int bits, int T) {
  DecodeMapShape m;
  m.piece_words = kUnitK * bits / 32 * (bits == 3 ? 2 : 1);
  m.code_rows = kRowsPerCta;
  m.code_pieces = kUnits / (bits == 3 ? 2 : 1);
  m.unit_k = kUnitK;
  m.x_tokens = T <= 8 ? 8 : 16;
  m.x_units = kUnits;
  return m;
}

cudaError_t launch_decode_gemm(const DecodeArgs& a, const CUtensorMap& tmC,
                               const CUtensorMap& tmX, cudaStream_t stream, bool pdl) {
  if (a.M == 0 || a.T == 0) return cudaSuccess;
  // 32-bit indexing inside the kernel
  if (a.T > 16 || a.K % (kUnitK * (a.bits == 3 ? 2 : 1)) != 0 || a.group < 32 ||
      (a.group & (a.group - 1)) != 0 ||
      a.K > (int64_t{1} << 30) || a.M > (int64_t{1} << 30) || a.r > (int64_t{1} << 20) ||
      a.ax_ld > (int64_t{1} << 20) || a.ldy > (int64_t{1} << 30))
    return cudaErrorInvalidValue;
  int gs = 0;
  while ((1 << (gs + 1)) <= a.group) ++gs;
  switch (a.bits) {
    case 2: return launch_decode_bits<2>(tmC, tmX, a, gs, stream, pdl);
    case 3: return launch_decode_bits<3>(tmC, tmX, a, gs, stream, pdl);
    case 4: return launch_decode_bits<4>(tmC, tmX, a, gs, stream, pdl);
    case 8: return launch_decode_bits<8>(tmC, tmX, a, gs, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}


AxMmaPlan ax_mma_plan(int64_t r, int64_t T, int64_t d) {
  // at up to 16 tokens the tensor-core GEMM's K splits measured faster
  // (8192 -> 28672 at one token: 118.9 against 121.2 us per forward)
  if (T <= 16 || T > kAxMaxTokens || r < 8 || r > 96 || r % 8 != 0) return {0, 0};
  const int kc = r <= 32 ? 512 : 256;
  return {static_cast<int>((d + kc - 1) / kc), kc};
}

cudaError_t launch_ax_mma(const void* A, const void* X, int64_t d, int64_t T, int64_t r,
                          const AxMmaPlan& plan, float* P, void* AX, int64_t ax_ld,
                          cudaStream_t stream, bool pdl) {
  if (T == 0) return cudaSuccess;
  if (plan.splits < 1 || (plan.splits > 1 && P == nullptr)) return cudaErrorInvalidValue;
  const auto* a = static_cast<const __nv_bfloat16*>(A);
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  auto* ax = static_cast<__nv_bfloat16*>(AX);
  const int kc = plan.kc;
  switch (r / 8) {
    case 1: return launch_ax_mma_nt<1>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 2: return launch_ax_mma_nt<2>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 3: return launch_ax_mma_nt<3>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 4: return launch_ax_mma_nt<4>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 5: return launch_ax_mma_nt<5>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 6: return launch_ax_mma_nt<6>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 7: return launch_ax_mma_nt<7>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 8: return launch_ax_mma_nt<8>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 9: return launch_ax_mma_nt<9>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 10: return launch_ax_mma_nt<10>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 11: return launch_ax_mma_nt<11>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    case 12: return launch_ax_mma_nt<12>(a, x, d, T, kc, plan.splits, P, ax, ax_ld, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ttq
