// Steps (2)-(3) of the TTQ layer for a few tokens (T <= 16):
//   Y[t][j] = sum_i s_jk (q_ji - z_jk) X'[t][i]  (+ sum_k B[j][k] AX[t][k])
// with X' = X D^(-1/2) in binary16 (gist.science/zh/paper/2603.19296,
// section 2.1 for W_hat, 2.2 for the static low-rank pair).
//
// With so few tokens the product is a matrix-vector product bound by the
// bytes of the packed codes, so the kernel is built to keep many of them in
// flight: one producer warp streams, per stage of 128 input channels, the
// code tile of the CTA's 64 rows of W and the matching 128 channels of X'
// into shared memory by TMA (8 stages deep); four consumer warps, 16 rows
// each, dequantise the codes in registers and feed them to warp-level
// tensor-core MMAs (m16n8k16, binary16 x binary16 -> fp32).  The weights never
// exist in binary16 outside registers.  The operand values are those the
// large-tile product forms: binary16 (1024 + q) - (1024 + z) is exact and
// the product with s rounds once.
//
// The order of the 16 products inside one MMA is free as long as the A and
// B operands agree on it, so each lane (g = lane / 4, c = lane % 4) owns 32
// contiguous channels of a stage -- its codes are one vector load from
// shared memory -- and pairs codes the way the packing makes cheap: INT4
// channels (i, i + 4) of a 16-channel unit come out of one word with one
// mask, INT2 (i, i + 8), INT3 (2i, 2i + 1).  The matching pairs of X' are
// put together with byte permutes.  Lanes with c >= 2 walk their two units
// in the opposite order, which together with the 128-byte swizzle of the X'
// tiles keeps the shared-memory reads free of bank conflicts.
//
// Register layout of m16n8k16 (PTX ISA, warp-level MMA): the A registers
// hold rows g and g + 8 at the lane's K pair 0 (registers 0, 1) and K pair 1
// (registers 2, 3); B holds the same two K pairs of column (token) g; C
// holds rows g, g + 8 at columns 2c, 2c + 1.
//
// Every barrier wait is bounded (1 s); a wait that gives up sets
// TTQ_FLAG_TIMEOUT, stops the CTA's other warps, lets the copies in flight
// land, and the CTA returns without storing Y.
#include <mutex>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kRowGroups = 4;                   // 16-row groups per CTA
constexpr int kRowsPerCta = 16 * kRowGroups;
constexpr int kConsumers = 2 * kRowGroups;      // x 2: even and odd stages
constexpr int kStageK = 128;                    // input channels per stage
constexpr int kStages = 8;

template <int BITS>
constexpr int stage_words() { return kStageK * BITS / 32; }   // code words per row and stage
template <int BITS>
constexpr uint32_t code_tile_bytes() { return kRowsPerCta * stage_words<BITS>() * 4; }
template <int NTT>
constexpr uint32_t xh_tile_bytes() { return 2u * 8u * NTT * 128u; }  // two 64-channel boxes
template <int BITS, int NTT>
constexpr uint32_t stage_bytes() {
  return (xh_tile_bytes<NTT>() + code_tile_bytes<BITS>() + 1023u) & ~1023u;
}
template <int BITS, int NTT>
constexpr size_t decode_smem_bytes() {
  return static_cast<size_t>(kStages) * stage_bytes<BITS, NTT>() + 1024;
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

// (m + q) - (m + z) on a binary16 pair (exact)
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t magic_pair, uint32_t zc2) {
  __half2 a, zc;
  memcpy(&a, &magic_pair, 4);
  memcpy(&zc, &zc2, 4);
  const __half2 v = __hsub2(a, zc);
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}

// s ((m + q) - (m + z)) on a binary16 pair
__device__ __forceinline__ uint32_t dequant_pair(uint32_t magic_pair, uint32_t zc2, uint32_t s2) {
  __half2 a, zc, s;
  memcpy(&a, &magic_pair, 4);
  memcpy(&zc, &zc2, 4);
  memcpy(&s, &s2, 4);
  const __half2 v = __hmul2(__hsub2(a, zc), s);
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
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

// The lane's code words of one row for the current stage (its 32 channels).
template <int BITS>
struct LaneCodes {
  uint32_t w[BITS];
};

template <int BITS>
__device__ __forceinline__ LaneCodes<BITS> load_lane_codes(uint32_t row_addr, int c) {
  LaneCodes<BITS> v;
  if (BITS == 4) {
    const uint4 a = lds128(row_addr + 16 * c);
    v.w[0] = a.x; v.w[1] = a.y; v.w[2 % BITS] = a.z; v.w[3 % BITS] = a.w;
  } else if (BITS == 2) {
    const uint2 a = lds64(row_addr + 8 * c);
    v.w[0] = a.x; v.w[1] = a.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) v.w[i] = lds32(row_addr + 12 * c + 4 * i);
  }
  return v;
}

// Code pairs of 16-channel unit uu of the lane's 32 channels as binary16
// pairs (m + q), m a power of two per pair, so that no shift is needed
// where the code bits already sit inside the significand: a code at bit b
// of a 16-bit half, OR-ed into the exponent of m = 2^(10 - b), reads m + q.
// INT4: P[i] = channels (i, i + 4), P[4 + i] = (8 + i, 12 + i); INT2: P[i] =
// (i, i + 8); INT3: P[i] = (2i, 2i + 1) (all with m = 1024).
// kind[i] = log2(m) of pair i.
template <int BITS>
struct PairSpec {
  static constexpr int kinds = BITS == 4 ? 2 : (BITS == 2 ? 5 : 1);
};
template <int BITS>
__device__ __forceinline__ constexpr int pair_kind(int i) {
  // index into the per-row table of (m + z): INT4 {1024, 64}; INT2 {1024,
  // 256, 64, 16, 4}; INT3 {1024}
  return BITS == 4 ? (i & 1) : (BITS == 2 ? (i < 5 ? i : i - 5) : 0);
}
__device__ __forceinline__ constexpr uint32_t kind_magic(int bits, int k) {
  return bits == 2 ? (k == 0 ? 0x64006400u : k == 1 ? 0x5C005C00u : k == 2 ? 0x54005400u
                                                 : k == 3 ? 0x4C004C00u : 0x44004400u)
                   : (k == 0 ? 0x64006400u : 0x54005400u);
}
template <int BITS>
__device__ __forceinline__ void magic_pairs(const LaneCodes<BITS>& v, int uu, uint32_t (&P)[8]) {
  if (BITS == 4) {
    const uint32_t lo = uu ? v.w[2 % BITS] : v.w[0];
    const uint32_t hi = uu ? v.w[3 % BITS] : v.w[1];
    const uint32_t lo8 = lo >> 8, hi8 = hi >> 8;
    P[0] = (lo & 0x000F000Fu) | 0x64006400u;    // channels 0, 4
    P[1] = (lo & 0x00F000F0u) | 0x54005400u;    // 1, 5
    P[2] = (lo8 & 0x000F000Fu) | 0x64006400u;   // 2, 6
    P[3] = (lo8 & 0x00F000F0u) | 0x54005400u;   // 3, 7
    P[4] = (hi & 0x000F000Fu) | 0x64006400u;
    P[5] = (hi & 0x00F000F0u) | 0x54005400u;
    P[6] = (hi8 & 0x000F000Fu) | 0x64006400u;
    P[7] = (hi8 & 0x00F000F0u) | 0x54005400u;
  } else if (BITS == 2) {
    const uint32_t w = uu ? v.w[1] : v.w[0];
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
    // unit 0: bits 0..47 of the lane's 96; unit 1: bits 48..95
    const uint64_t b = uu ? ((static_cast<uint64_t>(v.w[2 % BITS]) << 16) | (v.w[1] >> 16))
                          : (static_cast<uint64_t>(v.w[1] & 0xFFFFu) << 32 | v.w[0]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t t = static_cast<uint32_t>(b >> (6 * i));
      P[i] = (t & 0x7u) | ((t & 0x38u) << 13) | 0x64006400u;
    }
  }
}

// The X' pairs B[0..7] matching magic_pairs, from the unit's 16 channels
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

// PS: the quantisation group spans whole stages (group >= 128), so s is
// applied once per stage and row to the fp32 sum of (q - z) X' (exact
// operands); otherwise every operand is the binary16 s (q - z).
template <int BITS, int NTT, bool PS>
__global__ void __launch_bounds__(32 * (1 + kConsumers)) ttq_decode_kernel(
    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
    const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros, int64_t K,
    int64_t M, int64_t T, int group_shift, const __nv_bfloat16* __restrict__ Blr,
    const __nv_bfloat16* __restrict__ AX, int64_t r, int64_t ax_ld, void* __restrict__ Y,
    int64_t ldy, int y_f32, uint32_t* status) {
  extern __shared__ uint8_t dsm[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ int abort_s;
  __shared__ float red[kRowGroups][NTT][4][32];   // odd-stage sums
  constexpr uint32_t kXh = xh_tile_bytes<NTT>();
  constexpr uint32_t kCode = code_tile_bytes<BITS>();
  constexpr uint32_t kStage = stage_bytes<BITS, NTT>();
  constexpr int kKinds = PairSpec<BITS>::kinds;
  const uint32_t smem = (smem_addr(dsm) + 1023u) & ~1023u;
  uint8_t* smem_ptr = dsm + (smem - smem_addr(dsm));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nsteps = static_cast<int>((K + kStageK - 1) / kStageK);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  volatile int* abort_flag = &abort_s;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kRowGroups);
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
        tma_load_2d(&tmX, &full[s], base, st * kStageK, 0);
        tma_load_2d(&tmX, &full[s], base + kXh / 2, st * kStageK + 64, 0);
        tma_load_2d(&tmC, &full[s], base + kXh, st * stage_words<BITS>(),
                    static_cast<int32_t>(row0));
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
  // warp 1 + rg + 4 kpar: rows 16 rg .. 16 rg + 15 of the CTA, stages
  // kpar, kpar + 2, ...
  const int cw = warp - 1;
  const int rg = cw % kRowGroups;
  const int kpar = cw / kRowGroups;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int rla = 16 * rg + g, rlb = rla + 8;   // rows within the CTA
  const int64_t ra = row0 + rla, rb = row0 + rlb;
  const int64_t ngroups = K >> group_shift;
  const int64_t sra = (ra < M ? ra : M - 1) * ngroups;
  const int64_t srb = (rb < M ? rb : M - 1) * ngroups;
  // s | z << 16 of both rows for stage st (the lane's 32 channels lie in one
  // quantisation group); past K the group index is clamped (the matching X'
  // is zero)
  auto load_sz = [&](int st, uint32_t& za_s, uint32_t& zb_s) {
    int64_t gi = (static_cast<int64_t>(st) * kStageK + 32 * c) >> group_shift;
    if (gi >= ngroups) gi = ngroups - 1;
    za_s = static_cast<uint32_t>(__ldg(scales + sra + gi)) |
           (static_cast<uint32_t>(__ldg(zeros + sra + gi)) << 16);
    zb_s = static_cast<uint32_t>(__ldg(scales + srb + gi)) |
           (static_cast<uint32_t>(__ldg(zeros + srb + gi)) << 16);
  };
  const int my_n = (nsteps - kpar + 1) / 2;     // stages of this warp
  // the loads of s, z run kSzAhead stages ahead in a ring whose slot index
  // is static after unrolling (moving a register still being loaded would
  // wait for the load)
  constexpr int kSzAhead = 4;
  uint32_t sz_a[kSzAhead], sz_b[kSzAhead];
#pragma unroll
  for (int i = 0; i < kSzAhead; ++i) {
    sz_a[i] = sz_b[i] = 0u;
    if (i < my_n) load_sz(kpar + 2 * i, sz_a[i], sz_b[i]);
  }
  float acc[NTT][4];
#pragma unroll
  for (int tt = 0; tt < NTT; ++tt) acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;
  bool ok = true;
  const uint32_t xbox = static_cast<uint32_t>(c >> 1) * (kXh / 2);
  const uint32_t flip = static_cast<uint32_t>(c >> 1);

  for (int i0 = 0; i0 < my_n && ok; i0 += kSzAhead) {
#pragma unroll
    for (int j = 0; j < kSzAhead; ++j) {
      const int i = i0 + j;
      if (i >= my_n) break;
      const int st = kpar + 2 * i;
      const int s = st % kStages;
      const uint32_t ph = static_cast<uint32_t>(st / kStages) & 1u;
      int got = 1;
      if (lane == 0) got = mbar_wait(&full[s], ph, abort_flag) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        if (lane == 0) {
          *abort_flag = 1;
          set_flag(status, TTQ_FLAG_TIMEOUT);
        }
        ok = false;
        break;
      }
      const uint32_t base = smem + s * kStage;
      const uint32_t code_base = base + kXh;
      const LaneCodes<BITS> va =
          load_lane_codes<BITS>(code_base + rla * (stage_words<BITS>() * 4), c);
      const LaneCodes<BITS> vb =
          load_lane_codes<BITS>(code_base + rlb * (stage_words<BITS>() * 4), c);
      // (m + z) pairs of both rows for every magic m in use (exact), and s
      const __half za = __ushort_as_half(static_cast<uint16_t>(sz_a[j] >> 16));
      const __half zb = __ushort_as_half(static_cast<uint16_t>(sz_b[j] >> 16));
      uint32_t zca[kKinds], zcb[kKinds];
#pragma unroll
      for (int k = 0; k < kKinds; ++k) {
        const __half m = __ushort_as_half(static_cast<uint16_t>(kind_magic(BITS, k) & 0xFFFFu));
        zca[k] = static_cast<uint32_t>(__half_as_ushort(__hadd(za, m))) * 0x00010001u;
        zcb[k] = static_cast<uint32_t>(__half_as_ushort(__hadd(zb, m))) * 0x00010001u;
      }
      const uint32_t s2a = (sz_a[j] & 0xFFFFu) * 0x00010001u;
      const uint32_t s2b = (sz_b[j] & 0xFFFFu) * 0x00010001u;
      const float sfa = __half2float(__ushort_as_half(static_cast<uint16_t>(sz_a[j] & 0xFFFFu)));
      const float sfb = __half2float(__ushort_as_half(static_cast<uint16_t>(sz_b[j] & 0xFFFFu)));
      if (i + kSzAhead < my_n) load_sz(st + 2 * kSzAhead, sz_a[j], sz_b[j]);

      float part[NTT][4];
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt) part[tt][0] = part[tt][1] = part[tt][2] = part[tt][3] = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int uu = u ^ static_cast<int>(flip);
        uint32_t Pa[8], Pb[8];
        magic_pairs<BITS>(va, uu, Pa);
        magic_pairs<BITS>(vb, uu, Pb);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const int k = pair_kind<BITS>(p);
          if (PS) {
            Pa[p] = hsub2_bits(Pa[p], zca[k]);
            Pb[p] = hsub2_bits(Pb[p], zcb[k]);
          } else {
            Pa[p] = dequant_pair(Pa[p], zca[k], s2a);
            Pb[p] = dequant_pair(Pb[p], zcb[k], s2b);
          }
        }
        // the unit's 16 channels of X' are chunks 4 (c & 1) + 2 uu and the
        // next one of the 128-byte rows of box c >> 1, swizzled by row & 7
        const uint32_t ch0 = static_cast<uint32_t>(4 * (c & 1) + 2 * uu);
#pragma unroll
        for (int tt = 0; tt < NTT; ++tt) {
          const uint32_t rowa = base + xbox + static_cast<uint32_t>(8 * tt + g) * 128u;
          const uint4 x0 = lds128(rowa + ((ch0 ^ static_cast<uint32_t>(g)) << 4));
          const uint4 x1 = lds128(rowa + (((ch0 + 1) ^ static_cast<uint32_t>(g)) << 4));
          const uint32_t X[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint32_t B[8];
          x_pairs<BITS>(X, B);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t a[4] = {Pa[2 * k], Pb[2 * k], Pa[2 * k + 1], Pb[2 * k + 1]};
            mma_m16n8k16_f16(PS ? part[tt] : acc[tt], a, B[2 * k], B[2 * k + 1]);
          }
        }
      }
      if (PS) {
#pragma unroll
        for (int tt = 0; tt < NTT; ++tt) {
          acc[tt][0] = fmaf(sfa, part[tt][0], acc[tt][0]);
          acc[tt][1] = fmaf(sfa, part[tt][1], acc[tt][1]);
          acc[tt][2] = fmaf(sfb, part[tt][2], acc[tt][2]);
          acc[tt][3] = fmaf(sfb, part[tt][3], acc[tt][3]);
        }
      }
      (void)s2a;
      (void)s2b;
      (void)sfa;
      (void)sfb;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // the low-rank term B (A X), bf16 operands in the plain register layout
  // (K pair 0 = k 2c, 2c + 1; K pair 1 = k 2c + 8, 2c + 9), on the odd-stage
  // warps
  if (kpar == 1 && r > 0 && ok) {
    const bool ra_ok = ra < M, rb_ok = rb < M;
    const __nv_bfloat16* ba = Blr + (ra_ok ? ra : 0) * r;
    const __nv_bfloat16* bb = Blr + (rb_ok ? rb : 0) * r;
    for (int64_t k0 = 0; k0 < r; k0 += 16) {
      const int64_t kc = k0 + 2 * c;
      const bool lo_ok = kc < r, hi_ok = kc + 8 < r;
      uint32_t a[4];
      a[0] = (ra_ok && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc)) : 0u;
      a[1] = (rb_ok && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc)) : 0u;
      a[2] = (ra_ok && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc + 8)) : 0u;
      a[3] = (rb_ok && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc + 8)) : 0u;
#pragma unroll
      for (int tt = 0; tt < NTT; ++tt) {
        const int64_t n = 8 * tt + g;
        const bool n_ok = n < T;
        const __nv_bfloat16* axn = AX + (n_ok ? n : 0) * ax_ld;
        const uint32_t b0 = (n_ok && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc)) : 0u;
        const uint32_t b1 = (n_ok && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc + 8)) : 0u;
        mma_m16n8k16_bf16(acc[tt], a, b0, b1);
      }
    }
  }

  // the odd-stage warps hand their sums to the even-stage warps of the same
  // rows, which add them (a fixed order) and store Y: C rows g, g + 8 are
  // rows ra, rb; columns 2c, 2c + 1 of token tile tt are tokens 8 tt + 2c,
  // 8 tt + 2c + 1
  if (kpar == 1) {
#pragma unroll
    for (int tt = 0; tt < NTT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[rg][tt][e][lane] = acc[tt][e];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
  if (kpar == 1 || *abort_flag) return;
#pragma unroll
  for (int tt = 0; tt < NTT; ++tt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = acc[tt][e] + red[rg][tt][e][lane];
      const int64_t row = (e < 2) ? ra : rb;
      const int64_t t = 8 * tt + 2 * c + (e & 1);
      if (row < M && t < T) {
        if (y_f32) static_cast<float*>(Y)[t * ldy + row] = v;
        else static_cast<__nv_bfloat16*>(Y)[t * ldy + row] = __float2bfloat16_rn(v);
      }
    }
  }
}

template <int BITS, int NTT, bool PS>
cudaError_t launch_decode_typed(const CUtensorMap& tmC, const CUtensorMap& tmX,
                                const DecodeArgs& a, int group_shift, cudaStream_t stream,
                                bool pdl) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  constexpr size_t smem = decode_smem_bytes<BITS, NTT>();
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(ttq_decode_kernel<BITS, NTT, PS>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return attr_err;
  const dim3 grid(static_cast<unsigned>((a.M + kRowsPerCta - 1) / kRowsPerCta));
  return launch_kernel(ttq_decode_kernel<BITS, NTT, PS>, grid, dim3(32 * (1 + kConsumers)), smem,
                       stream, pdl, tmC, tmX, a.scales, a.zeros, a.K, a.M, a.T, group_shift,
                       static_cast<const __nv_bfloat16*>(a.Blr),
                       static_cast<const __nv_bfloat16*>(a.AX), a.r, a.ax_ld, a.Y, a.ldy,
                       a.y_f32 ? 1 : 0, a.status);
}

template <int BITS>
cudaError_t launch_decode_bits(const CUtensorMap& tmC, const CUtensorMap& tmX,
                               const DecodeArgs& a, int gs, cudaStream_t stream, bool pdl) {
  const bool ps = a.group >= kStageK;
  if (a.T > 8)
    return ps ? launch_decode_typed<BITS, 2, true>(tmC, tmX, a, gs, stream, pdl)
              : launch_decode_typed<BITS, 2, false>(tmC, tmX, a, gs, stream, pdl);
  return ps ? launch_decode_typed<BITS, 1, true>(tmC, tmX, a, gs, stream, pdl)
            : launch_decode_typed<BITS, 1, false>(tmC, tmX, a, gs, stream, pdl);
}

}  // namespace

int decode_code_box_words(int bits) { return kStageK * bits / 32; }
int decode_code_box_rows() { return kRowsPerCta; }

cudaError_t launch_decode_gemm(const DecodeArgs& a, const CUtensorMap& tmC,
                               const CUtensorMap& tmX, cudaStream_t stream, bool pdl) {
  if (a.M == 0 || a.T == 0) return cudaSuccess;
  if (a.T > 16 || a.K % 32 != 0 || a.group < 32 || (a.group & (a.group - 1)) != 0)
    return cudaErrorInvalidValue;
  int gs = 0;
  while ((1 << (gs + 1)) <= a.group) ++gs;
  switch (a.bits) {
    case 2: return launch_decode_bits<2>(tmC, tmX, a, gs, stream, pdl);
    case 3: return launch_decode_bits<3>(tmC, tmX, a, gs, stream, pdl);
    case 4: return launch_decode_bits<4>(tmC, tmX, a, gs, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ttq
