// Steps (2)-(3) of the TTQ layer in one pass over W, for a few tokens
// (T <= 16):
//   x = W_ji sqrt(D_i);  per group: s, z from the range of x;
//   q = clamp(rint(x / s) + z);  Y[t][j] = sum_i s (q - z) X'[t][i]
// with X' = X D^(-1/2) in binary16 (gist.science/zh/paper/2603.19296,
// section 2.1 for W_hat = Q[W D^{1/2}] D^{-1/2}, section 2.3 for the cost:
// at decode the 3d'd test-time term is the whole cost, so W is read once
// and nothing is written back but Y).  The codes are formed exactly as the
// quantiser forms them (same binary32 operations in the same order), and are
// stored only when the caller asks for them.
//
// Work: the weight is cut into units of 256 rows x 128 input channels; the
// units are numbered row-tile-major and every CTA takes one contiguous range
// of them (a persistent grid of one CTA per SM, equal shares), so no SM
// idles at the end.  A row tile whose units fall to two or more CTAs is
// finished by the last of them to arrive: each writes its partial sums to
// the workspace and takes a ticket, and the last adds the partials in CTA
// order (a fixed order: the result does not depend on timing).
//
// Per unit, lane 0 of warp 0 loads by TMA into one stage of a ring: the
// 256 x 128 tile of W (two 64-channel boxes, 128-byte swizzle), the unit's
// 128 channels of X' (two boxes, 8 or 16 tokens) and of sqrt(D).  Each of
// the 16 warps owns 16 rows of the tile; a stage is refilled once all of
// them have released it, which keeps them in step.  Lane (g, c) (g = lane / 4, c =
// lane % 4) holds rows pi(g) and pi(g) + 8 of the warp's 16 (pi(g) =
// g / 2 + 4 (g % 2), which keeps its shared-memory reads free of bank
// conflicts) and channels 8 (4m + c) .. + 7 for m = 0..3: a row's group
// range is the lane's own values plus two shuffles among its four lanes.
// The operand (1024 + q) - (1024 + z) = q - z is exact in binary16; the
// warp-level MMA (m16n8k16, binary16 x binary16 -> fp32) sums a group's
// products and s multiplies that fp32 sum once.  K positions of the MMA map
// to channels the same way for every lane with the same c, and X' is read
// with the same map, so the products pair up.
//
// Every mbarrier wait is bounded (1 s); a wait that gives up sets
// TTQ_FLAG_TIMEOUT, the CTA stops storing results, lets its copies in
// flight land and returns.  Its tickets are then left unbalanced: the
// caller re-initialises the workspace after a timeout.
#include <atomic>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kFdWarps = 16;
constexpr int kFdThreads = 32 * kFdWarps;
constexpr int kFdRows = 16 * kFdWarps;               // rows of W per unit
constexpr int kFdK = 128;                            // channels per unit
constexpr uint32_t kFdWBox = kFdRows * 64 * 2;       // one 64-channel box of W: 32 KiB

template <int NTT>
constexpr int fd_stages() { return 3; }
// X' box: 8 NTT tokens x 64 channels of binary16
template <int NTT>
constexpr uint32_t fd_x_box() { return 8u * NTT * 128u; }
template <int NTT>
constexpr uint32_t fd_stage_bytes() {
  return (2u * kFdWBox + 2u * fd_x_box<NTT>() + kFdK * 4u + 1023u) & ~1023u;
}
template <int NTT>
constexpr size_t fd_smem_bytes() {
  return static_cast<size_t>(fd_stages<NTT>()) * fd_stage_bytes<NTT>() + 1024;
}

struct FdDev {
  const float* Dh;        // sqrt(D) [K] float32 (source of the per-unit bulk copy)
  int K, M, T;
  int nsl;                // K / 128
  int64_t units;          // row tiles x nsl
  const __nv_bfloat16* Blr;
  const __nv_bfloat16* AX;
  int r, ax_ld;
  void* Y;
  int ldy, y_f32;
  uint32_t* codes;        // may be null (then scales, zeros are null too)
  uint16_t* scales;
  uint16_t* zeros;
  float* part;            // [gridDim.x][2][kFdWarps][32][4 NTT] partial sums
  uint32_t* tickets;      // [row tiles], zero before and after every call
  uint32_t* status;
};



__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float min3_nan(float a, float b, float c) {
  float r;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  __half2 x, y;
  memcpy(&x, &a, 4);
  memcpy(&y, &b, 4);
  const __half2 v = __hsub2(x, y);
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}

// Row of the warp's 16 that MMA row g (< 8) stands for (g + 8 stands for
// pi(g) + 8): rows read at once by a quarter warp then differ in bit 2, so
// their swizzled 16-byte chunks fall on distinct banks.
__device__ __forceinline__ int fd_pi(int g) { return (g >> 1) + 4 * (g & 1); }

// Address of 16-byte chunk j (0..15) of row R in two 64-column boxes of
// `rows` rows each, 128-byte swizzle (row R of a box at (R/8)*1024 +
// (R%8)*128, chunk jj of the row XOR-ed with R%8).
__device__ __forceinline__ uint32_t sw_chunk(uint32_t base, uint32_t box_bytes, int R, int j) {
  const int jj = j & 7;
  return base + static_cast<uint32_t>(j >> 3) * box_bytes + static_cast<uint32_t>(R >> 3) * 1024u +
         static_cast<uint32_t>(R & 7) * 128u + (static_cast<uint32_t>(jj ^ (R & 7)) << 4);
}

// Group parameters of one row's group with range [mn, mx] (mn <= 0 <= mx),
// in the quantiser's binary32 order: s, 1/s from the significand table,
// and z.  zc: binary16 1024 + z in both halves; zz: 0x6400 + z in both
// 16-bit lanes (the clamp bound of the codes is 0x6400 + 2^b - 1).
template <int BITS>
struct GroupQ {
  float sf, inv;
  uint32_t zz;
  uint16_t s16, z;
  bool bad, ovf;
};
template <int BITS>
__device__ __forceinline__ GroupQ<BITS> group_params(float mn, float mx, const float* rcp) {
  constexpr int QMAX = (1 << BITS) - 1;
  GroupQ<BITS> p;
  const float range = __fsub_rn(mx, mn);
  p.bad = !(range <= 3.402823466e38f);
  float s32 = div_by_const<QMAX>(range);
  if (!(s32 >= 6.103515625e-05f)) s32 = 6.103515625e-05f;  // 2^-14
  const __half s16 = __float2half_ru(s32);
  p.sf = __half2float(s16);
  const uint32_t sbits = __half_as_ushort(s16);
  const int sexp = static_cast<int>((sbits >> 10) & 31u) - 15;
  p.inv = __int_as_float(__float_as_int(rcp[sbits & 1023u]) - sexp * (1 << 23));
  const int zi = __float_as_int(__fmaf_rn(-mn, p.inv, 12582912.0f)) - 0x4B400000;
  const int z = min(max(zi, 0), QMAX);
  p.z = static_cast<uint16_t>(z);
  p.zz = (0x6400u + static_cast<uint32_t>(z)) * 0x00010001u;
  p.s16 = static_cast<uint16_t>(sbits);
  p.ovf = static_cast<bool>(__hisinf(s16)) || p.sf * static_cast<float>(QMAX) > 65504.f;
  return p;
}

// Four code pairs of one 8-channel chunk as binary16 (1024 + q) pairs:
// rint of the exact product x * inv (one fused multiply-add with
// 1.5 * 2^23), plus 0x6400 + z, clamped at 0x6400 + 2^b - 1 (a finite
// group never needs the lower clamp).
template <int BITS>
__device__ __forceinline__ void chunk_codes(const float2 (&x)[4], float inv, uint32_t zz,
                                            uint32_t (&qh)[4]) {
  constexpr uint32_t QQ = (0x6400u + static_cast<uint32_t>((1 << BITS) - 1)) * 0x00010001u;
  const float2 inv2 = make_float2(inv, inv);
  const float2 magic2 = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 r = __ffma2_rn(x[p], inv2, magic2);
    qh[p] = __viaddmin_s16x2(__byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410), zz, QQ);
  }
}

// Stores the 8 codes of one chunk (channels ch .. ch + 7 of row `row`) into
// the packed LSB-first stream: 8 * BITS bits at bit BITS * ch.
template <int BITS>
__device__ __forceinline__ void store_chunk_codes(uint32_t* codes, int64_t wpr, int64_t row,
                                                  int ch, const uint32_t (&qh)[4]) {
  uint32_t v = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    v |= ((qh[p] & 0xFFu)) << (BITS * 2 * p);
    v |= ((qh[p] >> 16) & 0xFFu) << (BITS * (2 * p + 1));
  }
  // (1024 + q) has q in its low bits: 0x6400 + q with q < 16 keeps q in the
  // low byte, and the shifts above drop the 0x64 of the high byte
  uint8_t* rowp = reinterpret_cast<uint8_t*>(codes + row * wpr);
  const int64_t bit = static_cast<int64_t>(BITS) * ch;   // a multiple of 8 * BITS
  if (BITS == 4) {
    *reinterpret_cast<uint32_t*>(rowp + bit / 8) = v;
  } else if (BITS == 2) {
    *reinterpret_cast<uint16_t*>(rowp + bit / 8) = static_cast<uint16_t>(v);
  } else {
    rowp[bit / 8] = static_cast<uint8_t>(v);
    rowp[bit / 8 + 1] = static_cast<uint8_t>(v >> 8);
    rowp[bit / 8 + 2] = static_cast<uint8_t>(v >> 16);
  }
}

template <int BITS, int NTT, int GROUP, bool CODES>
__global__ void __launch_bounds__(kFdThreads, 1) ttq_fused_decode_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
    const FdDev a) {
  constexpr int kStages = fd_stages<NTT>();
  constexpr uint32_t kXBox = fd_x_box<NTT>();
  constexpr uint32_t kStage = fd_stage_bytes<NTT>();
  constexpr uint32_t kStageTx = 2u * kFdWBox + 2u * kXBox + kFdK * 4u;
  constexpr int NG = kFdK / GROUP;         // groups per unit row
  constexpr int MPG = 4 / NG;              // chunk steps m per group
  extern __shared__ uint8_t dsm[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ float rcp_sig[1024];
  __shared__ int abort_s;
  __shared__ int last_s;
  const uint32_t smem = (smem_addr(dsm) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int c = lane & 3;
  volatile int* abort_flag = &abort_s;

  const int64_t U = a.units;
  const int64_t NC = gridDim.x;
  const int64_t u_begin = U * blockIdx.x / NC;
  const int64_t u_end = U * (blockIdx.x + 1) / NC;

  const bool producer = threadIdx.x == 0;
  auto issue_w = [&](int64_t u, int s) {
    const int64_t tile = u / a.nsl;
    const int32_t k0 = static_cast<int32_t>((u - tile * a.nsl) * kFdK);
    const int32_t r0 = static_cast<int32_t>(tile * kFdRows);
    const uint32_t base = smem + static_cast<uint32_t>(s) * kStage;
    mbar_arrive_expect_tx(&full[s], kStageTx);
    tma_load_2d(&tmW, &full[s], dsm + (base - smem_addr(dsm)), k0, r0);
    tma_load_2d(&tmW, &full[s], dsm + (base + kFdWBox - smem_addr(dsm)), k0 + 64, r0);
  };
  auto issue_xh = [&](int64_t u, int s) {
    const int64_t tile = u / a.nsl;
    const int32_t k0 = static_cast<int32_t>((u - tile * a.nsl) * kFdK);
    const uint32_t base = smem + static_cast<uint32_t>(s) * kStage + 2u * kFdWBox;
    tma_load_2d(&tmX, &full[s], dsm + (base - smem_addr(dsm)), k0, 0);
    tma_load_2d(&tmX, &full[s], dsm + (base + kXBox - smem_addr(dsm)), k0 + 64, 0);
    bulk_load(base + 2u * kXBox, a.Dh + k0, kFdK * 4u, &full[s]);
  };
  const int64_t n_units = u_end - u_begin;
  // only the first stage is requested at launch: every CTA asks at once, and
  // a CTA's first stage lands sooner when it does not compete with the
  // others' second and third; those follow once it has landed
  const int first_issue = n_units > 0 ? 1 : 0;
  const int ring_fill = static_cast<int>(n_units < kStages ? n_units : kStages);
  if (producer) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFdWarps);
    }
    abort_s = 0;
    last_s = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    // the weight does not depend on the kernels before this one: the first
    // stages' W boxes are requested before anything else
    for (int i = 0; i < first_issue; ++i) issue_w(u_begin + i, i);
  }
  // binary32 1 / (1 + k/1024) for the binary16 significands (1/s of a
  // normal binary16 s = m 2^e is this times 2^-e, exactly)
  for (int k = threadIdx.x; k < 1024; k += kFdThreads)
    rcp_sig[k] = __fdiv_rn(1.0f, 1.0f + static_cast<float>(k) * 0.0009765625f);
  __syncthreads();
  allow_dependents_launch();
  grid_dependency_wait();
  if (producer)
    for (int i = 0; i < first_issue; ++i) issue_xh(u_begin + i, i);
  int64_t issued = first_issue;   // units requested so far (producer only)

  // rows of this lane in the unit tile, and its MMA accumulators
  const int rA = 16 * warp + fd_pi(g);   // MMA row g
  const int rB = rA + 8;                 // MMA row g + 8
  float acc[NTT][4];
#pragma unroll
  for (int t = 0; t < NTT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  bool bad = false, ovf = false;
  const int64_t wpr = static_cast<int64_t>(a.K) * BITS / 32;
  const int ngroups = a.K / GROUP;

  for (int64_t u = u_begin; u < u_end; ++u) {
    const int i = static_cast<int>(u - u_begin);
    const int s = i % kStages;
    const uint32_t ph = static_cast<uint32_t>(i / kStages) & 1u;
    const int64_t tile = u / a.nsl;
    const int sl = static_cast<int>(u - tile * a.nsl);
    // refill: the slot of unit i - 1 takes unit i - 1 + kStages once every
    // warp has finished with it
    if (producer && i >= 1 && issued < n_units && *abort_flag == 0) {
      const int sp = (i - 1) % kStages;
      if (mbar_wait(&empty[sp], static_cast<uint32_t>((i - 1) / kStages) & 1u, abort_flag)) {
        issue_w(u_begin + issued, sp);
        issue_xh(u_begin + issued, sp);
        ++issued;
      } else {
        *abort_flag = 1;
        set_flag(a.status, TTQ_FLAG_TIMEOUT);
      }
    }
    bool ok = *abort_flag == 0;
    if (ok) {
      if (!mbar_wait(&full[s], ph, abort_flag)) {
        if (lane == 0) {
          *abort_flag = 1;
          set_flag(a.status, TTQ_FLAG_TIMEOUT);
        }
        ok = false;
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (producer && i == 0 && ok) {
      for (int k = 1; k < ring_fill; ++k) {
        issue_w(u_begin + k, k);
        issue_xh(u_begin + k, k);
      }
      issued = ring_fill;
    }
    if (ok) {
      const uint32_t base = smem + static_cast<uint32_t>(s) * kStage;
      const uint32_t xbase = base + 2u * kFdWBox;
      const uint32_t hbase = xbase + 2u * kXBox;
      // x = W * sqrt(D) for the lane's 2 rows x 4 chunks of 8 channels
      float2 xa[4][4], xb[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = 4 * m + c;
        const uint4 h0 = lds128(hbase + 32u * j);
        const uint4 h1 = lds128(hbase + 32u * j + 16u);
        const float hv[8] = {__uint_as_float(h0.x), __uint_as_float(h0.y), __uint_as_float(h0.z),
                             __uint_as_float(h0.w), __uint_as_float(h1.x), __uint_as_float(h1.y),
                             __uint_as_float(h1.z), __uint_as_float(h1.w)};
        const uint4 wa = lds128(sw_chunk(base, kFdWBox, rA, j));
        const uint4 wb = lds128(sw_chunk(base, kFdWBox, rB, j));
        const uint32_t wav[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t wbv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 hp = make_float2(hv[2 * p], hv[2 * p + 1]);
          xa[m][p] = __fmul2_rn(make_float2(__uint_as_float(wav[p] << 16),
                                            __uint_as_float(wav[p] & 0xFFFF0000u)), hp);
          xb[m][p] = __fmul2_rn(make_float2(__uint_as_float(wbv[p] << 16),
                                            __uint_as_float(wbv[p] & 0xFFFF0000u)), hp);
        }
      }
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        // the group's range, per row: the lane's chunks, then its 4 lanes
        float mna = 0.f, mxa = 0.f, mnb = 0.f, mxb = 0.f;
#pragma unroll
        for (int mm = 0; mm < MPG; ++mm) {
          const int m = gi * MPG + mm;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            mna = min3_nan(mna, xa[m][p].x, xa[m][p].y);
            mxa = max3_nan(mxa, xa[m][p].x, xa[m][p].y);
            mnb = min3_nan(mnb, xb[m][p].x, xb[m][p].y);
            mxb = max3_nan(mxb, xb[m][p].x, xb[m][p].y);
          }
        }
        // The lanes of a pair (c, c ^ 1) split the two rows: even c takes
        // row A, odd c row B.  Each hands the other the range of the row it
        // does not take, the pair (c, c ^ 2) completes the range, each lane
        // computes its row's s, 1/s and z, and the pair swaps them.
        const bool keep_a = (c & 1) == 0;
        float kmn = min_nan(keep_a ? mna : mnb,
                            __shfl_xor_sync(0xffffffffu, keep_a ? mnb : mna, 1));
        float kmx = max_nan(keep_a ? mxa : mxb,
                            __shfl_xor_sync(0xffffffffu, keep_a ? mxb : mxa, 1));
        kmn = min_nan(kmn, __shfl_xor_sync(0xffffffffu, kmn, 2));
        kmx = max_nan(kmx, __shfl_xor_sync(0xffffffffu, kmx, 2));
        const GroupQ<BITS> qk = group_params<BITS>(kmn, kmx, rcp_sig);
        bad |= qk.bad;
        ovf |= qk.ovf;
        GroupQ<BITS> qo;   // the partner's row
        qo.sf = __shfl_xor_sync(0xffffffffu, qk.sf, 1);
        qo.inv = __shfl_xor_sync(0xffffffffu, qk.inv, 1);
        qo.zz = __shfl_xor_sync(0xffffffffu, qk.zz, 1);
        {
          const uint32_t sz = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(qk.s16) |
                                                               (static_cast<uint32_t>(qk.z) << 16), 1);
          qo.s16 = static_cast<uint16_t>(sz & 0xFFFFu);
          qo.z = static_cast<uint16_t>(sz >> 16);
        }
        const GroupQ<BITS>& qa = keep_a ? qk : qo;
        const GroupQ<BITS>& qb = keep_a ? qo : qk;
        const uint32_t za = (0x6400u + qa.z) * 0x00010001u;
        const uint32_t zb = (0x6400u + qb.z) * 0x00010001u;
        float part[NTT][4];
#pragma unroll
        for (int t = 0; t < NTT; ++t) part[t][0] = part[t][1] = part[t][2] = part[t][3] = 0.f;
#pragma unroll
        for (int mm = 0; mm < MPG; ++mm) {
          const int m = gi * MPG + mm;
          const int j = 4 * m + c;
          uint32_t qa4[4], qb4[4];
          chunk_codes<BITS>(xa[m], qa.inv, qa.zz, qa4);
          chunk_codes<BITS>(xb[m], qb.inv, qb.zz, qb4);
          if (CODES) {
            const int64_t rowa = tile * kFdRows + rA, rowb = tile * kFdRows + rB;
            const int ch = sl * kFdK + 8 * j;
            if (rowa < a.M) store_chunk_codes<BITS>(a.codes, wpr, rowa, ch, qa4);
            if (rowb < a.M) store_chunk_codes<BITS>(a.codes, wpr, rowb, ch, qb4);
          }
          uint32_t opa[4], opb[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            opa[p] = hsub2_bits(qa4[p], za);   // q - z, exact
            opb[p] = hsub2_bits(qb4[p], zb);
          }
          // X' of tokens (column g of each 8-token tile), this chunk
#pragma unroll
          for (int t = 0; t < NTT; ++t) {
            const uint4 xv = lds128(sw_chunk(xbase, kXBox, 8 * t + fd_pi(g), j));
            const uint32_t A0[4] = {opa[0], opb[0], opa[1], opb[1]};
            const uint32_t A1[4] = {opa[2], opb[2], opa[3], opb[3]};
            mma_f16(part[t], A0, xv.x, xv.y);
            mma_f16(part[t], A1, xv.z, xv.w);
          }
        }
        // s of row rA applies to C rows g (elements 0, 1), s of rB to g + 8
#pragma unroll
        for (int t = 0; t < NTT; ++t) {
          acc[t][0] = fmaf(qa.sf, part[t][0], acc[t][0]);
          acc[t][1] = fmaf(qa.sf, part[t][1], acc[t][1]);
          acc[t][2] = fmaf(qb.sf, part[t][2], acc[t][2]);
          acc[t][3] = fmaf(qb.sf, part[t][3], acc[t][3]);
        }
        if (CODES && c == 0) {
          const int gidx = (sl * kFdK + gi * GROUP) / GROUP;
          const int64_t rowa = tile * kFdRows + rA, rowb = tile * kFdRows + rB;
          const uint16_t za16 = __half_as_ushort(__int2half_rn(qa.z));
          const uint16_t zb16 = __half_as_ushort(__int2half_rn(qb.z));
          if (rowa < a.M) {
            a.scales[rowa * ngroups + gidx] = qa.s16;
            a.zeros[rowa * ngroups + gidx] = za16;
          }
          if (rowb < a.M) {
            a.scales[rowb * ngroups + gidx] = qb.s16;
            a.zeros[rowb * ngroups + gidx] = zb16;
          }
        }
      }
    }
    // this warp is done with the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    // ------------------------------------------------ end of a row tile
    const bool tile_end = sl == a.nsl - 1 || u + 1 == u_end;
    if (!tile_end) continue;
    const int64_t t_first = tile * a.nsl, t_last = t_first + a.nsl - 1;
    // CTAs that own units of this tile (CTA c covers [U c / NC, U (c+1) / NC))
    const int64_t c_first = ((t_first + 1) * NC - 1) / U;
    const int64_t c_last = ((t_last + 1) * NC - 1) / U;
    const bool alive = *abort_flag == 0;
    bool finish = c_first == c_last;   // the whole tile is this CTA's
    if (!finish) {
      // publish this CTA's partial sums; the last CTA to arrive finishes.
      // Slot 1 holds the tile the range starts inside of, slot 0 the tile
      // it ends inside of (a CTA has at most one of each).
      const int slot = u_begin <= t_first ? 0 : 1;
      float* pp = a.part + ((static_cast<int64_t>(blockIdx.x) * 2 + slot) * kFdWarps + warp) * 32 * 4 * NTT;
#pragma unroll
      for (int t = 0; t < NTT; ++t)
        __stcg(reinterpret_cast<float4*>(pp) + t * 32 + lane,
               make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]));
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        int last = 0;
        if (alive) {
          const uint32_t prev = atomicAdd(a.tickets + tile, 1u);
          last = prev == static_cast<uint32_t>(c_last - c_first) ? 1 : 0;
          if (last) a.tickets[tile] = 0u;   // ready for the next call
        }
        last_s = last;
      }
      __syncthreads();
      finish = last_s != 0;
      if (finish) {
        __threadfence();
#pragma unroll
        for (int t = 0; t < NTT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        for (int64_t cc = c_first; cc <= c_last; ++cc) {
          const int sl2 = (U * cc / NC) <= t_first ? 0 : 1;
          const float* qp =
              a.part + ((cc * 2 + sl2) * kFdWarps + warp) * 32 * 4 * NTT;
#pragma unroll
          for (int t = 0; t < NTT; ++t) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(qp) + t * 32 + lane);
            acc[t][0] += v.x;
            acc[t][1] += v.y;
            acc[t][2] += v.z;
            acc[t][3] += v.w;
          }
        }
      }
    }
    if (finish && alive) {
      const int64_t rowa = tile * kFdRows + rA, rowb = tile * kFdRows + rB;
      // the static low-rank term B (A X) for the lane's rows: bf16 MMAs,
      // C rows g / g + 8 = rows rowa / rowb, columns = tokens 8 t + pi(col)
      if (a.r > 0) {
        for (int k0 = 0; k0 < a.r; k0 += 16) {
          const int kc = k0 + 2 * c;
          const bool lo_ok = kc < a.r, hi_ok = kc + 8 < a.r;
          const __nv_bfloat16* ba = a.Blr + (rowa < a.M ? rowa : 0) * static_cast<int64_t>(a.r);
          const __nv_bfloat16* bb = a.Blr + (rowb < a.M ? rowb : 0) * static_cast<int64_t>(a.r);
          uint32_t A[4];
          A[0] = (rowa < a.M && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc)) : 0u;
          A[1] = (rowb < a.M && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc)) : 0u;
          A[2] = (rowa < a.M && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(ba + kc + 8)) : 0u;
          A[3] = (rowb < a.M && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(bb + kc + 8)) : 0u;
#pragma unroll
          for (int t = 0; t < NTT; ++t) {
            const int n = 8 * t + fd_pi(g);   // token of MMA column g
            const bool n_ok = n < a.T;
            const __nv_bfloat16* axn = a.AX + static_cast<int64_t>(n_ok ? n : 0) * a.ax_ld;
            const uint32_t b0 = (n_ok && lo_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc)) : 0u;
            const uint32_t b1 = (n_ok && hi_ok) ? __ldg(reinterpret_cast<const uint32_t*>(axn + kc + 8)) : 0u;
            mma_bf16(acc[t], A, b0, b1);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NTT; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t row = (e >> 1) ? rowb : rowa;
          const int tok = 8 * t + fd_pi(2 * c + (e & 1));
          if (row < a.M && tok < a.T) {
            const int64_t at = static_cast<int64_t>(tok) * a.ldy + row;
            if (a.y_f32) static_cast<float*>(a.Y)[at] = acc[t][e];
            else static_cast<__nv_bfloat16*>(a.Y)[at] = __float2bfloat16_rn(acc[t][e]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NTT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  }

  if (__any_sync(0xffffffffu, ovf) && lane == 0)
    set_flag(a.status, TTQ_FLAG_NONFINITE | TTQ_FLAG_SCALE_OVERFLOW);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_flag(a.status, TTQ_FLAG_NONFINITE);
  if (producer && *abort_flag) {
    // the copies still in flight land before the CTA's shared memory goes
    // away (waited on with a fresh limit, not cut short by the abort)
    int never = 0;
    for (int64_t k = issued > kStages ? issued - kStages : 0; k < issued; ++k) {
      const int kk = static_cast<int>(k);
      mbar_wait(&full[kk % kStages], static_cast<uint32_t>(kk / kStages) & 1u, &never);
    }
  }
}

template <int BITS, int NTT, int GROUP, bool CODES>
cudaError_t launch_fd_typed(const CUtensorMap& tmW, const CUtensorMap& tmX, const FdDev& a,
                            int grid, cudaStream_t stream, bool pdl) {
  constexpr size_t smem = fd_smem_bytes<NTT>();
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e = cudaFuncSetAttribute(ttq_fused_decode_kernel<BITS, NTT, GROUP, CODES>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_relaxed);
  }
  return launch_kernel(ttq_fused_decode_kernel<BITS, NTT, GROUP, CODES>, dim3(grid), dim3(kFdThreads),
                       smem, stream, pdl, tmW, tmX, a);
}

template <int BITS, int NTT, int GROUP>
cudaError_t launch_fd_codes(const CUtensorMap& tmW, const CUtensorMap& tmX, const FdDev& a,
                            int grid, cudaStream_t stream, bool pdl) {
  if (a.codes != nullptr) return launch_fd_typed<BITS, NTT, GROUP, true>(tmW, tmX, a, grid, stream, pdl);
  return launch_fd_typed<BITS, NTT, GROUP, false>(tmW, tmX, a, grid, stream, pdl);
}

template <int BITS, int NTT>
cudaError_t launch_fd_group(int group, const CUtensorMap& tmW, const CUtensorMap& tmX,
                            const FdDev& a, int grid, cudaStream_t stream, bool pdl) {
  switch (group) {
    case 32: return launch_fd_codes<BITS, NTT, 32>(tmW, tmX, a, grid, stream, pdl);
    case 64: return launch_fd_codes<BITS, NTT, 64>(tmW, tmX, a, grid, stream, pdl);
    case 128: return launch_fd_codes<BITS, NTT, 128>(tmW, tmX, a, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS>
cudaError_t launch_fd_bits(int group, const CUtensorMap& tmW, const CUtensorMap& tmX,
                           const FdDev& a, int grid, cudaStream_t stream, bool pdl) {
  if (a.T > 8) return launch_fd_group<BITS, 2>(group, tmW, tmX, a, grid, stream, pdl);
  return launch_fd_group<BITS, 1>(group, tmW, tmX, a, grid, stream, pdl);
}

}  // namespace

FusedDecodePlan fused_decode_plan(int64_t dp, int64_t d, int64_t T) {
  FusedDecodePlan p;
  p.row_tiles = (dp + kFdRows - 1) / kFdRows;
  p.units = p.row_tiles * (d / kFdK);
  // one CTA per SM (its 16 warps share one ring, so none races ahead of the
  // others as a second CTA on the SM would), and never more CTAs than
  // units: every CTA then owns at least one unit, so the CTAs that share a
  // row tile are consecutive and all take its ticket
  p.grid = static_cast<int>(p.units < kFusedDecodePlanSMs ? p.units : kFusedDecodePlanSMs);
  if (p.grid < 1) p.grid = 1;
  p.part_floats = static_cast<int64_t>(p.grid) * 2 * kFdWarps * 32 * 4 * (T > 8 ? 2 : 1);
  return p;
}

int fused_decode_rows() { return kFdRows; }

bool fused_decode_supported(int64_t dp, int64_t d, int64_t T, int bits, int group) {
  return T >= 1 && T <= 16 && dp >= 1 && d >= kFdK && d % kFdK == 0 && bits >= 2 && bits <= 4 &&
         (group == 32 || group == 64 || group == 128) &&
         (dp + kFdRows - 1) / kFdRows <= kFusedDecodeMaxTiles && d <= (int64_t{1} << 30) &&
         dp <= (int64_t{1} << 30);
}

cudaError_t launch_fused_decode(const FusedDecodeArgs& a, const CUtensorMap& tmW,
                                const CUtensorMap& tmX, cudaStream_t stream, bool pdl) {
  if (!fused_decode_supported(a.M, a.K, a.T, a.bits, a.group)) return cudaErrorInvalidValue;
  if ((a.codes == nullptr) != (a.scales == nullptr) || (a.codes == nullptr) != (a.zeros == nullptr))
    return cudaErrorInvalidValue;
  const FusedDecodePlan plan = fused_decode_plan(a.M, a.K, a.T);
  FdDev g;
  g.Dh = a.Dh;
  g.K = static_cast<int>(a.K);
  g.M = static_cast<int>(a.M);
  g.T = static_cast<int>(a.T);
  g.nsl = static_cast<int>(a.K / kFdK);
  g.units = plan.units;
  g.Blr = static_cast<const __nv_bfloat16*>(a.Blr);
  g.AX = static_cast<const __nv_bfloat16*>(a.AX);
  g.r = static_cast<int>(a.r);
  g.ax_ld = static_cast<int>(a.ax_ld);
  g.Y = a.Y;
  g.ldy = static_cast<int>(a.ldy);
  g.y_f32 = a.y_f32 ? 1 : 0;
  g.codes = a.codes;
  g.scales = a.scales;
  g.zeros = a.zeros;
  g.part = a.part;
  g.tickets = a.tickets;
  g.status = a.status;
  switch (a.bits) {
    case 2: return launch_fd_bits<2>(a.group, tmW, tmX, g, plan.grid, stream, pdl);
    case 3: return launch_fd_bits<3>(a.group, tmW, tmX, g, plan.grid, stream, pdl);
    case 4: return launch_fd_bits<4>(a.group, tmW, tmX, g, plan.grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ttq
