// Step (2) of the TTQ layer without the final rescale: codes, scales and
// zeros of Q[W D^{1/2}] (gist.science/zh/paper/2603.19296, section 2.1),
// with Q the group-wise asymmetric scale + zero-point quantiser (blog.lo0.es
// "Test-time quantization ...", section "The maths that matter").
//
// The arithmetic follows one fixed binary32 order so that the codes match
// the CPU oracle bit for bit:
//   h = sqrt(D_i); x = W_ji * h; m = min(0, min x); M = max(0, max x);
//   s32 = (M - m) / (2^b - 1), floored at 2^-14; s = binary16 round-up(s32);
//   inv = 1 / s; z = clamp(rint(-m * inv)); q = clamp(rint(x * inv) + z),
// where the two products inside rint are exact (one fused multiply-add
// rounds them straight to the integer).  The quotient s32 is the correctly
// rounded one, formed by div_by_const (a product with the rounded
// reciprocal and one exact correction).  Every other operation is an
// explicitly rounded intrinsic, so no contraction can change a result.
//
// Layout of the work: a block owns a tile of `cw` consecutive input channels
// and walks rows of W with a grid stride.  A thread owns 16 consecutive
// channels (two 16-byte loads of bf16 W), keeps their sqrt(D) in registers
// for every row it visits, and the group's g/16 threads reduce min/max with
// shuffles.  A lane's 16 codes fill two words (INT4), one word (INT2) or 48
// bits (INT3: an even/odd lane pair makes 3 words).  Pairs of weights go
// through the packed f32x2 multiply, which rounds each lane exactly like the
// scalar one (checked on B200 against __fmul_rn).
// The kernel is HBM-bound: it reads W once and writes d*b/8 + 4d/g bytes per
// row.
#include <cuda_fp8.h>

#include <atomic>
#include <cstring>

#include <type_traits>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kThreads = 256;

// 16 consecutive weights of one row, kept packed until they are used.
template <typename WT>
struct Raw16;
template <>
struct Raw16<__nv_bfloat16> {
  uint4 v[2];
};
template <>
struct Raw16<float> {
  float4 v[4];
};

__device__ __forceinline__ void load16(const __nv_bfloat16* src, Raw16<__nv_bfloat16>& r) {
  r.v[0] = __ldcs(reinterpret_cast<const uint4*>(src));
  r.v[1] = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
}
__device__ __forceinline__ void load16(const float* src, Raw16<float>& r) {
#pragma unroll
  for (int i = 0; i < 4; ++i) r.v[i] = __ldcs(reinterpret_cast<const float4*>(src) + i);
}
__device__ __forceinline__ void zero16(Raw16<__nv_bfloat16>& r) {
  r.v[0] = r.v[1] = make_uint4(0u, 0u, 0u, 0u);
}
__device__ __forceinline__ void zero16(Raw16<float>& r) {
#pragma unroll
  for (int i = 0; i < 4; ++i) r.v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ void unpack16(const Raw16<__nv_bfloat16>& r, float2 (&x)[8]) {
  const uint32_t w[8] = {r.v[0].x, r.v[0].y, r.v[0].z, r.v[0].w, r.v[1].x, r.v[1].y, r.v[1].z, r.v[1].w};
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}
__device__ __forceinline__ void unpack16(const Raw16<float>& r, float2 (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = make_float2(r.v[i].x, r.v[i].y);
    x[2 * i + 1] = make_float2(r.v[i].z, r.v[i].w);
  }
}

__device__ __forceinline__ __half2 u32_as_half2(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return h;
}
__device__ __forceinline__ uint32_t half2_as_u32(__half2 h) {
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}

// Codes 4k..4k+3 (each < 16) from two pairs of 16-bit lanes a = (q0, q1),
// b = (q2, q3), as four 4-bit fields in the low 16 bits: a + b * 256 holds
// q0 | q2 << 8 and q1 | q3 << 8 in its lanes, and OR-ing it with itself
// shifted right by 12 brings q1 and q3 down to bits 4 and 12.
__device__ __forceinline__ uint32_t nibbles4(uint32_t a, uint32_t b) {
  const uint32_t t = a + (b << 8);
  return t | (t >> 12);
}
// The same for codes < 4: four 2-bit fields in the low byte.
__device__ __forceinline__ uint32_t crumbs4(uint32_t a, uint32_t b) {
  const uint32_t t = a + (b << 4);
  return t | (t >> 14);
}

// Three-input minimum / maximum that return NaN if any input is NaN (so a
// NaN weight reaches the group's range and is flagged there).
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

// With WQ the kernel also writes the dequantised weight s (q - z) as
// binary16 [dp][d] (wq), formed exactly as the product's A operand is
// formed from the codes: (1024 + q) - (1024 + z) is exact in binary16 and
// the product with s is rounded once.
// With SYM the symmetric quantiser: the scale covers max|x| with levels
// +-(2^(b-1) - 1) and the zero point is the constant 2^(b-1), so the stored
// (code, scale, zero) triples dequantise exactly as the asymmetric ones.
template <typename WT, int BITS, bool WQ, bool SYM>
__global__ void __launch_bounds__(kThreads, 2) qdq_pack_kernel(
    const WT* __restrict__ W, int64_t dp, int64_t d, const float* __restrict__ D, int group,
    int cw, uint32_t* __restrict__ codes, __half* __restrict__ scales,
    __half* __restrict__ zeros, __half* __restrict__ wq, uint32_t* __restrict__ status) {
  constexpr int QMAX = (1 << BITS) - 1;                     // largest code
  constexpr int QSPAN = SYM ? (1 << (BITS - 1)) - 1 : QMAX;  // levels the scale spans
  const int tpr = cw >> 4;            // threads per row of the tile (16 weights each)
  const int rpi = kThreads / tpr;     // rows per iteration of the block
  const int tx = threadIdx.x % tpr;
  const int ty = threadIdx.x / tpr;
  const int lane = threadIdx.x & 31;
  const int gthreads = group >> 4;    // threads sharing one group (2..16)
  const int64_t col = static_cast<int64_t>(blockIdx.x) * cw + tx * 16;
  const int64_t ngroups = d / group;
  const int64_t kgroup = col / group;  // this thread's group within the row
  const int64_t wpr = d * BITS / 32;   // words per row
  allow_dependents_launch();

  // the first rows of W do not depend on the previous kernel: load them
  // before waiting for it (D does)
  constexpr int kRows = 4;
  const int64_t step = static_cast<int64_t>(gridDim.y) * rpi;
  const int64_t stride = kRows * step;
  Raw16<WT> cur[kRows], nxt[kRows];
  auto load_rows = [&](int64_t b, Raw16<WT>(&dst)[kRows]) {
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int64_t row = b + u * step + ty;
      if (row < dp) load16(W + row * d + col, dst[u]);
      else zero16(dst[u]);
    }
  };
  if (static_cast<int64_t>(blockIdx.y) * rpi < dp) load_rows(static_cast<int64_t>(blockIdx.y) * rpi, cur);
  grid_dependency_wait();

  float2 h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    h[i] = D != nullptr ? make_float2(__fsqrt_rn(__ldg(D + col + 2 * i)), __fsqrt_rn(__ldg(D + col + 2 * i + 1)))
                        : make_float2(1.f, 1.f);
  float hchk = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) hchk += h[i].x + h[i].y;
  bool bad = !(hchk <= 3.402823466e38f);
  bool ovf = false;
  // binary32(1 / m) for the 1024 binary16 significands m = 1 + k/1024; the
  // reciprocal of a normal binary16 s = m 2^e is then this value times
  // 2^-e, exactly (a power-of-two scaling in the normal range)
  __shared__ float rcp_sig[1024];
  for (int k = threadIdx.x; k < 1024; k += kThreads)
    rcp_sig[k] = __fdiv_rn(1.0f, 1.0f + static_cast<float>(k) * 0.0009765625f);
  __syncthreads();

  // The loop bound is block-uniform so every lane takes part in the
  // shuffles; rows past the end are computed on zeros and not stored.  The
  // next kRows rows are loaded while the current ones are quantised.
  // quantise the kRows rows held in `buf`, starting at row b
  auto process = [&](int64_t b, const Raw16<WT>(&buf)[kRows]) {
    const int64_t base = b;
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int64_t row = base + u * step + ty;
        const bool active = row < dp;
        float2 x[8];
        unpack16(buf[u], x);
        float mn = 0.f, mx = 0.f;
  #pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[i] = __fmul2_rn(x[i], h[i]);
          mn = min3_nan(mn, x[i].x, x[i].y);
          mx = max3_nan(mx, x[i].x, x[i].y);
        }
        for (int o = gthreads >> 1; o > 0; o >>= 1) {
          mn = min_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const float range = __fsub_rn(mx, mn);
        bad |= !(range <= 3.402823466e38f);  // a NaN or infinite x, or a range beyond binary32
        // asymmetric: the range [m, M] over 2^b - 1 steps; symmetric: max|x|
        // over 2^(b-1) - 1 steps
        const float span = SYM ? max_nan(mx, -mn) : range;
        float s32 = div_by_const<QSPAN>(span);
        if (!(s32 >= 6.103515625e-05f)) s32 = 6.103515625e-05f;  // 2^-14
        const __half s16 = __float2half_ru(s32);
        const float s = __half2float(s16);
        // inv = binary32(1 / s) from the significand table and the exponent
        // (s >= 2^-14 is normal; an infinite s is flagged below)
        const uint32_t sbits = __half_as_ushort(s16);
        const int sexp = static_cast<int>((sbits >> 10) & 31u) - 15;
        const float inv = __int_as_float(__float_as_int(rcp_sig[sbits & 1023u]) - sexp * (1 << 23));
        // rint of the exact product x * inv: a fused multiply-add with
        // 1.5 * 2^23 rounds the true product to an integer, ties to even, for
        // |x * inv| < 2^22 (here |x * inv| <= 2^b + 1); the integer is read
        // from the low fraction bits.  For a finite group rint(x * inv) + z
        // is never below 0 (x >= m and rint is odd), so only the top is
        // clamped.
        const int zi = __float_as_int(__fmaf_rn(-mn, inv, 12582912.0f)) - 0x4B400000;
        const int z = SYM ? (1 << (BITS - 1)) : min(max(zi, 0), QMAX);
        // the 16 codes as eight (q_2i, q_2i+1) pairs of 16-bit lanes:
        // rint(x * inv) from the low bits of the fused multiply-add, plus z,
        // clamped at the top (one packed add-and-min per pair)
        const uint32_t zz = static_cast<uint32_t>(z) * 0x00010001u;
        constexpr uint32_t QQ = static_cast<uint32_t>(QMAX) * 0x00010001u;
        const float2 inv2 = make_float2(inv, inv);
        const float2 magic2 = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
        uint32_t qp[8];
  #pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 r = __ffma2_rn(x[i], inv2, magic2);
          const uint32_t n = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);
          qp[i] = __viaddmin_s16x2(n, zz, QQ);
        }
        if (WQ && active) {
          // s (q - z): (1024 + q) - (1024 + z) is exact in binary16, the
          // product with s rounds once
          const __half2 zc2 = u32_as_half2((0x6400u | static_cast<uint32_t>(z)) * 0x00010001u);
          const __half2 s2 = __half2half2(s16);
          uint32_t wh[8];
  #pragma unroll
          for (int i = 0; i < 8; ++i)
            wh[i] = half2_as_u32(__hmul2(__hsub2(u32_as_half2(qp[i] | 0x64006400u), zc2), s2));
          uint4* dst = reinterpret_cast<uint4*>(wq + row * d + col);
          dst[0] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          dst[1] = make_uint4(wh[4], wh[5], wh[6], wh[7]);
        }
        // s (q - z) alone is wanted when codes is null (the forward's
        // materialised weight): the packing and the stores below are skipped
        // (a grid-uniform branch, so the INT3 shuffles stay uniform)
        const bool want_codes = codes != nullptr;
        if (active && (tx & (gthreads - 1)) == 0) {
          // s (q - z) is formed in binary16 by the product: |q - z| <= 2^b - 1
          ovf |= static_cast<bool>(__hisinf(s16)) || s * static_cast<float>(QSPAN) > 65504.f;
        }
        if (!want_codes) continue;
        uint32_t lo = 0, hi = 0;  // INT4: codes 0-7 and 8-15; INT3: 24 bits each
        if (BITS == 4) {
          lo = __byte_perm(nibbles4(qp[0], qp[1]), nibbles4(qp[2], qp[3]), 0x5410);
          hi = __byte_perm(nibbles4(qp[4], qp[5]), nibbles4(qp[6], qp[7]), 0x5410);
        } else if (BITS == 2) {
          lo = __byte_perm(__byte_perm(crumbs4(qp[0], qp[1]), crumbs4(qp[2], qp[3]), 0x0040),
                           __byte_perm(crumbs4(qp[4], qp[5]), crumbs4(qp[6], qp[7]), 0x0040), 0x5410);
        } else {
  #pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t pair = (qp[i] & 0xFFFFu) | ((qp[i] >> 16) << BITS);
            if (i < 4) lo |= pair << (2 * BITS * i);
            else hi |= pair << (2 * BITS * (i - 4));
          }
        }
        if (active && (tx & (gthreads - 1)) == 0) {
          scales[row * ngroups + kgroup] = s16;
          zeros[row * ngroups + kgroup] =
              __hsub(__ushort_as_half(static_cast<uint16_t>(0x6400u | z)), __ushort_as_half(0x6400));
        }
        // the lane's 16 codes are 16*BITS bits at bit 16*BITS*(col/16)
        if (BITS == 4) {
          if (active) *reinterpret_cast<uint2*>(codes + row * wpr + (col >> 3)) = make_uint2(lo, hi);
        } else if (BITS == 2) {
          if (active) codes[row * wpr + (col >> 4)] = lo;
        } else {
          // 48 bits per lane; an even/odd lane pair makes 3 words
          const uint32_t a = lo | (hi << 24);  // bits 0-31
          const uint32_t b = hi >> 8;          // bits 32-47
          const uint32_t oa = __shfl_down_sync(0xffffffffu, a, 1);
          const uint32_t ob = __shfl_down_sync(0xffffffffu, b, 1);
          if (active && (tx & 1) == 0) {
            uint32_t* dst = codes + row * wpr + (col >> 5) * 3;
            dst[0] = a;
            dst[1] = b | (oa << 16);
            dst[2] = (oa >> 16) | (ob << 16);
          }
        }
      }
  };
  // ping-pong between two buffers (loop unrolled twice): the loads for the
  // next rows are in flight while the current ones are quantised
  int64_t base = static_cast<int64_t>(blockIdx.y) * rpi;
  for (; base < dp; base += 2 * stride) {
    if (base + stride < dp) load_rows(base + stride, nxt);
    process(base, cur);
    if (base + stride >= dp) break;
    if (base + 2 * stride < dp) load_rows(base + 2 * stride, cur);
    process(base + stride, nxt);
  }
  if (__any_sync(0xffffffffu, ovf) && lane == 0)
    set_flag(status, TTQ_FLAG_NONFINITE | TTQ_FLAG_SCALE_OVERFLOW);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_flag(status, TTQ_FLAG_NONFINITE);
}

// The scale, its reciprocal and the zero point of one group of one row from
// the group's range [mn, mx], in the quantiser's binary32 order (the same
// operations as qdq_pack_kernel), and whether the group is bad (a NaN or
// infinite x, or a range beyond binary32) or its scale overflows what the
// product forms in binary16.
template <int BITS, bool SYM>
struct GroupParams {
  uint32_t sz;   // binary16 bits of s in the high half, z in the low half
  float inv;     // binary32(1 / s)
  bool bad, ovf;
};
template <int BITS, bool SYM>
__device__ __forceinline__ GroupParams<BITS, SYM> group_params(float mn, float mx,
                                                               const float* rcp_sig) {
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int QSPAN = SYM ? (1 << (BITS - 1)) - 1 : QMAX;  // levels the scale spans
  GroupParams<BITS, SYM> g;
  const float range = __fsub_rn(mx, mn);
  g.bad = !(range <= 3.402823466e38f);
  const float span = SYM ? max_nan(mx, -mn) : range;
  float s32 = div_by_const<QSPAN>(span);
  if (!(s32 >= 6.103515625e-05f)) s32 = 6.103515625e-05f;  // 2^-14
  const __half s16 = __float2half_ru(s32);
  const float s = __half2float(s16);
  const uint32_t sbits = __half_as_ushort(s16);
  const int sexp = static_cast<int>((sbits >> 10) & 31u) - 15;
  g.inv = __int_as_float(__float_as_int(rcp_sig[sbits & 1023u]) - sexp * (1 << 23));
  const int zi = __float_as_int(__fmaf_rn(-mn, g.inv, 12582912.0f)) - 0x4B400000;
  const int z = SYM ? (1 << (BITS - 1)) : min(max(zi, 0), QMAX);
  g.sz = (sbits << 16) | static_cast<uint32_t>(z);
  g.ovf = static_cast<bool>(__hisinf(s16)) || s * static_cast<float>(QSPAN) > 65504.f;
  return g;
}

// The same quantiser for bf16 W, with W staged in shared memory.  Block
// (bx, by) owns the tile of cw channels at bx * cw and the row batches by,
// by + gridDim.y, ... of kStageRows * rpi consecutive rows (32 KiB of W).
// Thread (tx, ty) quantises rows ty, ty + rpi, ... of each batch, 16
// channels each, as in qdq_pack_kernel.  A batch lands in one stage of a
// ring of kQStages by one bulk copy per row segment, on the stage's
// mbarrier (bounded waits).  Each warp copies its rows of a stage into
// registers and releases the stage at once; the last warp to release it
// (a shared-memory count) posts the next batch's byte count and issues its
// copies, so the ring is refilled as soon as its data sits in registers
// and no warp waits for another.  With no rows of W held in registers
// between batches a thread keeps the four rows' scaled weights at once, and
// the G = group/16 lanes of a group reduce the four rows' ranges together:
// the first shuffle round (partner li ^ G/2) leaves each lane two rows
// (lane bit G/2 picks the pair), the second (li ^ G/4) one row, and the
// remaining rounds reduce that row.  Each lane then computes s, 1/s and z of
// its own row only (with G = 2, of its two rows), and the four rows' values
// are shuffled back to every lane of the group.  min and max are exact, so
// no result depends on the order.
constexpr int kStageRows = 4;   // rows per thread per batch
constexpr int kQStages = 3;
constexpr uint32_t kQStageBytes = kStageRows * kThreads * 16 * 2;   // 32 KiB
constexpr uint32_t kQSmemBytes = kQStages * kQStageBytes;           // 96 KiB

template <int BITS, bool WQ, bool SYM, int G>
__global__ void __launch_bounds__(kThreads, 2) qdq_stage_kernel(
    const __grid_constant__ CUtensorMap tmW, int w_box, const __nv_bfloat16* __restrict__ W,
    int64_t dp, int64_t d, const float* __restrict__ D, int cw, uint32_t* __restrict__ codes,
    __half* __restrict__ scales, __half* __restrict__ zeros, __half* __restrict__ wq,
    uint32_t* __restrict__ status) {
  static_assert(G == 2 || G == 4 || G == 8 || G == 16, "group of 32 to 256 channels");
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int kWarps = kThreads / 32;
  extern __shared__ __align__(128) uint8_t stage_smem[];   // [kQStages][rows][cw] bf16
  __shared__ __align__(8) uint64_t full[kQStages];
  __shared__ int released[kQStages];   // warps done with the stage's current batch
  __shared__ int issued_s;             // batches requested so far
  __shared__ int timeout_s;
  __shared__ float rcp_sig[1024];

  const int tpr = cw >> 4;            // threads per row (16 channels each)
  const int rpi = kThreads / tpr;     // rows per step of the block
  const int rows_pb = kStageRows * rpi;
  const uint32_t row_bytes = static_cast<uint32_t>(cw) * 2u;
  const int tx = threadIdx.x % tpr;
  const int ty = threadIdx.x / tpr;
  const int lane = threadIdx.x & 31;
  const int li = lane & (G - 1);      // lane within the group
  const int gbase = lane - li;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * cw;
  const int64_t col = col0 + tx * 16;
  const int64_t ngroups = d / (16 * G);
  const int64_t kgroup = col / (16 * G);
  const int64_t wpr = d * BITS / 32;
  const int64_t nb_all = (dp + rows_pb - 1) / rows_pb;
  const int64_t nb = blockIdx.y < nb_all ? (nb_all - blockIdx.y + gridDim.y - 1) / gridDim.y : 0;
  const uint32_t smem0 = smem_addr(stage_smem);
  allow_dependents_launch();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0;
    }
    fence_barrier_init();
    issued_s = static_cast<int>(nb < kQStages ? nb : kQStages);
    timeout_s = 0;
  }
  __syncthreads();
  // batch i of this block into stage i % kQStages (all lanes of one warp)
  auto issue = [&](int64_t i) {
    const int s = static_cast<int>(i % kQStages);
    const int64_t r0 = (blockIdx.y + i * gridDim.y) * rows_pb;
    if (w_box) {
      // one tensor-map box of rows_pb rows x cw channels (a whole stage;
      // rows past dp arrive as zeros and count toward the bytes)
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kQStageBytes);
        tma_load_2d(&tmW, &full[s], stage_smem + static_cast<size_t>(s) * kQStageBytes,
                    static_cast<int32_t>(col0), static_cast<int32_t>(r0));
      }
      return;
    }
    const int nrows = static_cast<int>(min(static_cast<int64_t>(rows_pb), dp - r0));
    if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nrows) * row_bytes);
    __syncwarp();
    const uint32_t dst = smem0 + static_cast<uint32_t>(s) * kQStageBytes;
    for (int r = lane; r < nrows; r += 32)
      bulk_load(dst + static_cast<uint32_t>(r) * row_bytes, W + (r0 + r) * d + col0, row_bytes,
                &full[s]);
  };
  // W does not depend on the previous kernel: the first batches are
  // requested before waiting for it (D does)
  if (threadIdx.x < 32)
    for (int64_t i = 0; i < nb && i < kQStages; ++i) issue(i);
  grid_dependency_wait();

  float2 h[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    h[k] = D != nullptr ? make_float2(__fsqrt_rn(__ldg(D + col + 2 * k)), __fsqrt_rn(__ldg(D + col + 2 * k + 1)))
                        : make_float2(1.f, 1.f);
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 8; ++k) bad |= !(h[k].x <= 3.402823466e38f) || !(h[k].y <= 3.402823466e38f);
  bool ovf = false;
  for (int k = threadIdx.x; k < 1024; k += kThreads)
    rcp_sig[k] = __fdiv_rn(1.0f, 1.0f + static_cast<float>(k) * 0.0009765625f);
  __syncthreads();

  const bool want_codes = codes != nullptr;
  const int pa = (li & (G / 2)) != 0 ? 1 : 0;              // row pair after the first shuffle round
  const int pb = G >= 4 && (li & (G / 4)) != 0 ? 1 : 0;    // row of the pair after the second
  int never = 0;
  for (int64_t i = 0; i < nb; ++i) {
    const int s = static_cast<int>(i % kQStages);
    const uint32_t ph = static_cast<uint32_t>(i / kQStages) & 1u;
    // warp-uniform (the work below shuffles)
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, &never))) {
      if (lane == 0) {
        set_flag(status, TTQ_FLAG_TIMEOUT);
        timeout_s = 1;
      }
      break;
    }
    const int64_t r0 = (blockIdx.y + i * gridDim.y) * rows_pb;
    const uint32_t base = smem0 + static_cast<uint32_t>(s) * kQStageBytes +
                          static_cast<uint32_t>(tx) * 32u;
    // the four rows' scaled weights and ranges (rows past dp hold stale
    // data: their results are never stored or flagged)
    float2 x[kStageRows][8];
    float mn[kStageRows], mx[kStageRows];
#pragma unroll
    for (int u = 0; u < kStageRows; ++u) {
      const uint32_t a = base + static_cast<uint32_t>(u * rpi + ty) * row_bytes;
      Raw16<__nv_bfloat16> raw;
      raw.v[0] = lds128(a);
      raw.v[1] = lds128(a + 16u);
      unpack16(raw, x[u]);
      mn[u] = 0.f;
      mx[u] = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        x[u][k] = __fmul2_rn(x[u][k], h[k]);
        mn[u] = min3_nan(mn[u], x[u][k].x, x[u][k].y);
        mx[u] = max3_nan(mx[u], x[u][k].x, x[u][k].y);
      }
    }
    // this warp is done with stage s (the fence orders its reads before the
    // bulk copies that will overwrite it); the last warp to say so refills it
    fence_proxy_async_smem();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(&released[s], 1) == kWarps - 1;
    if (__shfl_sync(0xffffffffu, last, 0)) {
      if (lane == 0) released[s] = 0;
      if (i + kQStages < nb) {
        if (lane == 0) issued_s = static_cast<int>(i + kQStages + 1);
        issue(i + kQStages);
      }
    }
    // first shuffle round (partner li ^ G/2): keep the row pair pa, send the other
    float kmn[2], kmx[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float smn = pa ? mn[j] : mn[2 + j];
      const float smx = pa ? mx[j] : mx[2 + j];
      kmn[j] = min_nan(pa ? mn[2 + j] : mn[j], __shfl_xor_sync(0xffffffffu, smn, G / 2));
      kmx[j] = max_nan(pa ? mx[2 + j] : mx[j], __shfl_xor_sync(0xffffffffu, smx, G / 2));
    }
    uint32_t psz[kStageRows];
    float pinv[kStageRows];
    if constexpr (G == 2) {
      // each lane holds the complete ranges of rows 2 pa and 2 pa + 1
      GroupParams<BITS, SYM> gp[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        gp[j] = group_params<BITS, SYM>(kmn[j], kmx[j], rcp_sig);
        const int64_t row = r0 + (2 * pa + j) * rpi + ty;
        if (row < dp) {
          bad |= gp[j].bad;
          ovf |= gp[j].ovf;
          if (want_codes) {
            scales[row * ngroups + kgroup] = __ushort_as_half(static_cast<uint16_t>(gp[j].sz >> 16));
            zeros[row * ngroups + kgroup] =
                __hsub(__ushort_as_half(static_cast<uint16_t>(0x6400u | (gp[j].sz & 0xFFFFu))),
                       __ushort_as_half(0x6400));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kStageRows; ++u) {
        psz[u] = __shfl_sync(0xffffffffu, gp[u & 1].sz, gbase + (u >> 1));
        pinv[u] = __shfl_sync(0xffffffffu, gp[u & 1].inv, gbase + (u >> 1));
      }
    } else {
      // second shuffle round (partner li ^ G/4): keep row 2 pa + pb
      const float smn = pb ? kmn[0] : kmn[1];
      const float smx = pb ? kmx[0] : kmx[1];
      float rmn = min_nan(pb ? kmn[1] : kmn[0], __shfl_xor_sync(0xffffffffu, smn, G / 4));
      float rmx = max_nan(pb ? kmx[1] : kmx[0], __shfl_xor_sync(0xffffffffu, smx, G / 4));
#pragma unroll
      for (int o = G / 8; o > 0; o >>= 1) {
        rmn = min_nan(rmn, __shfl_xor_sync(0xffffffffu, rmn, o));
        rmx = max_nan(rmx, __shfl_xor_sync(0xffffffffu, rmx, o));
      }
      const GroupParams<BITS, SYM> gp = group_params<BITS, SYM>(rmn, rmx, rcp_sig);
      const int64_t row = r0 + (2 * pa + pb) * rpi + ty;
      if (row < dp) {
        bad |= gp.bad;
        ovf |= gp.ovf;
        // one lane per row stores its scale and zero
        if (want_codes && (li & (G / 4 - 1)) == 0) {
          scales[row * ngroups + kgroup] = __ushort_as_half(static_cast<uint16_t>(gp.sz >> 16));
          zeros[row * ngroups + kgroup] =
              __hsub(__ushort_as_half(static_cast<uint16_t>(0x6400u | (gp.sz & 0xFFFFu))),
                     __ushort_as_half(0x6400));
        }
      }
#pragma unroll
      for (int u = 0; u < kStageRows; ++u) {
        const int src = gbase + (u >> 1) * (G / 2) + (u & 1) * (G / 4);
        psz[u] = __shfl_sync(0xffffffffu, gp.sz, src);
        pinv[u] = __shfl_sync(0xffffffffu, gp.inv, src);
      }
    }

#pragma unroll
    for (int u = 0; u < kStageRows; ++u) {
      const int64_t row = r0 + u * rpi + ty;
      const bool active = row < dp;
      const uint32_t z = psz[u] & 0xFFFFu;
      // codes as in qdq_pack_kernel: rint(x * inv) from the fused
      // multiply-add with 1.5 * 2^23, plus z, clamped at the top
      const uint32_t zz = z * 0x00010001u;
      constexpr uint32_t QQ = static_cast<uint32_t>(QMAX) * 0x00010001u;
      const float2 inv2 = make_float2(pinv[u], pinv[u]);
      const float2 magic2 = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
      uint32_t qp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 r = __ffma2_rn(x[u][k], inv2, magic2);
        const uint32_t n = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);
        qp[k] = __viaddmin_s16x2(n, zz, QQ);
      }
      if (WQ && active) {
        const __half2 zc2 = u32_as_half2((0x6400u | z) * 0x00010001u);
        const __half2 s2 = u32_as_half2((psz[u] >> 16) * 0x00010001u);
        uint32_t wh[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          wh[k] = half2_as_u32(__hmul2(__hsub2(u32_as_half2(qp[k] | 0x64006400u), zc2), s2));
        uint4* dst = reinterpret_cast<uint4*>(wq + row * d + col);
        dst[0] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        dst[1] = make_uint4(wh[4], wh[5], wh[6], wh[7]);
      }
      if (!want_codes) continue;
      uint32_t lo = 0, hi = 0;
      if (BITS == 4) {
        lo = __byte_perm(nibbles4(qp[0], qp[1]), nibbles4(qp[2], qp[3]), 0x5410);
        hi = __byte_perm(nibbles4(qp[4], qp[5]), nibbles4(qp[6], qp[7]), 0x5410);
      } else if (BITS == 2) {
        lo = __byte_perm(__byte_perm(crumbs4(qp[0], qp[1]), crumbs4(qp[2], qp[3]), 0x0040),
                         __byte_perm(crumbs4(qp[4], qp[5]), crumbs4(qp[6], qp[7]), 0x0040), 0x5410);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t pair = (qp[k] & 0xFFFFu) | ((qp[k] >> 16) << BITS);
          if (k < 4) lo |= pair << (2 * BITS * k);
          else hi |= pair << (2 * BITS * (k - 4));
        }
      }
      if (BITS == 4) {
        if (active) *reinterpret_cast<uint2*>(codes + row * wpr + (col >> 3)) = make_uint2(lo, hi);
      } else if (BITS == 2) {
        if (active) codes[row * wpr + (col >> 4)] = lo;
      } else {
        const uint32_t a = lo | (hi << 24);
        const uint32_t bw = hi >> 8;
        const uint32_t oa = __shfl_down_sync(0xffffffffu, a, 1);
        const uint32_t ob = __shfl_down_sync(0xffffffffu, bw, 1);
        if (active && (tx & 1) == 0) {
          uint32_t* dst = codes + row * wpr + (col >> 5) * 3;
          dst[0] = a;
          dst[1] = bw | (oa << 16);
          dst[2] = (oa >> 16) | (ob << 16);
        }
      }
    }
  }
  __syncthreads();
  if (timeout_s && threadIdx.x == 0) {
    // a wait gave up: let the copies still in flight land before the block
    // exits (the latest batch of each stage, each with a fresh limit)
    for (int64_t k = issued_s - kQStages; k < issued_s; ++k)
      if (k >= 0) mbar_wait(&full[k % kQStages], static_cast<uint32_t>(k / kQStages) & 1u, &never);
  }
  if (__any_sync(0xffffffffu, ovf) && lane == 0)
    set_flag(status, TTQ_FLAG_NONFINITE | TTQ_FLAG_SCALE_OVERFLOW);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_flag(status, TTQ_FLAG_NONFINITE);
}

// FP8 (E4M3) codes with the activation-aware scale (blog.lo0.es, the
// comparison with FP8 end to end: TTQ derives s, the code format is free):
//   x = W_ji sqrt(D_i); s32 = max|x| / 448, floored at 2^-14;
//   s = binary16 round-up(s32); inv = 1 / s;
//   code = E4M3 round-to-nearest-even, saturating at +-448, of the binary32
//          product x * inv (the sign of a product that rounds to 0 is kept);
//   zero = +0;  reconstruction s * e4m3(code).
// Layout as in qdq_pack_kernel (16 consecutive channels per thread, the
// group's threads reduce the range with shuffles); the 16 one-byte codes
// of a thread are one 16-byte store.  With WQ the kernel also writes the
// binary16 s * e4m3(code) (the E4M3 value converts to binary16 exactly; the
// product with s rounds once); with WQ and codes == nullptr it writes that
// alone (no codes, scales or zeros).
template <typename WT, bool WQ>
__global__ void __launch_bounds__(kThreads, 2) qdq_fp8_kernel(
    const WT* __restrict__ W, int64_t dp, int64_t d, const float* __restrict__ D, int group,
    int cw, uint32_t* __restrict__ codes, __half* __restrict__ scales,
    __half* __restrict__ zeros, __half* __restrict__ wq, uint32_t* __restrict__ status) {
  const int tpr = cw >> 4;
  const int rpi = kThreads / tpr;
  const int tx = threadIdx.x % tpr;
  const int ty = threadIdx.x / tpr;
  const int lane = threadIdx.x & 31;
  const int gthreads = group >> 4;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * cw + tx * 16;
  const int64_t ngroups = d / group;
  const int64_t kgroup = col / group;
  const int64_t wpr = d / 4;            // four one-byte codes per word
  allow_dependents_launch();
  constexpr int kRows = 4;
  const int64_t step = static_cast<int64_t>(gridDim.y) * rpi;
  const int64_t stride = kRows * step;
  Raw16<WT> cur[kRows], nxt[kRows];
  auto load_rows = [&](int64_t b, Raw16<WT>(&dst)[kRows]) {
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int64_t row = b + u * step + ty;
      if (row < dp) load16(W + row * d + col, dst[u]);
      else zero16(dst[u]);
    }
  };
  if (static_cast<int64_t>(blockIdx.y) * rpi < dp) load_rows(static_cast<int64_t>(blockIdx.y) * rpi, cur);
  grid_dependency_wait();

  float2 h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    h[i] = D != nullptr ? make_float2(__fsqrt_rn(__ldg(D + col + 2 * i)), __fsqrt_rn(__ldg(D + col + 2 * i + 1)))
                        : make_float2(1.f, 1.f);
  float hchk = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) hchk += h[i].x + h[i].y;
  bool bad = !(hchk <= 3.402823466e38f);
  bool ovf = false;
  // binary32(1 / m) for the binary16 significands m = 1 + k/1024 (see
  // qdq_pack_kernel)
  __shared__ float rcp_sig[1024];
  for (int k = threadIdx.x; k < 1024; k += kThreads)
    rcp_sig[k] = __fdiv_rn(1.0f, 1.0f + static_cast<float>(k) * 0.0009765625f);
  __syncthreads();

  auto process = [&](int64_t b, const Raw16<WT>(&buf)[kRows]) {
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int64_t row = b + u * step + ty;
      const bool active = row < dp;
      float2 x[8];
      unpack16(buf[u], x);
      float mn = 0.f, mx = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[i] = __fmul2_rn(x[i], h[i]);
        mn = min3_nan(mn, x[i].x, x[i].y);
        mx = max3_nan(mx, x[i].x, x[i].y);
      }
      for (int o = gthreads >> 1; o > 0; o >>= 1) {
        mn = min_nan(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      bad |= !(__fsub_rn(mx, mn) <= 3.402823466e38f);
      const float amax = max_nan(mx, -mn);                 // max |x| of the group
      float s32 = div_by_const<448>(amax);
      if (!(s32 >= 6.103515625e-05f)) s32 = 6.103515625e-05f;  // 2^-14
      const __half s16 = __float2half_ru(s32);
      const float s = __half2float(s16);
      const uint32_t sbits = __half_as_ushort(s16);
      const int sexp = static_cast<int>((sbits >> 10) & 31u) - 15;
      const float inv = __int_as_float(__float_as_int(rcp_sig[sbits & 1023u]) - sexp * (1 << 23));
      const float2 inv2 = make_float2(inv, inv);
      // eight E4M3 pairs (channel 2i in the low byte), two per word
      uint32_t pr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pr[i] = static_cast<uint32_t>(
            __nv_cvt_float2_to_fp8x2(__fmul2_rn(x[i], inv2), __NV_SATFINITE, __NV_E4M3));
      if (active && codes != nullptr) {
        *reinterpret_cast<uint4*>(codes + row * wpr + (col >> 2)) =
            make_uint4(pr[0] | (pr[1] << 16), pr[2] | (pr[3] << 16), pr[4] | (pr[5] << 16),
                       pr[6] | (pr[7] << 16));
      }
      if (WQ && active) {
        const __half2 s2 = __half2half2(s16);
        uint32_t wh[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const __half2_raw r2 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pr[i]), __NV_E4M3);
          wh[i] = half2_as_u32(__hmul2(u32_as_half2(static_cast<uint32_t>(r2.x) | (static_cast<uint32_t>(r2.y) << 16)), s2));
        }
        uint4* dst = reinterpret_cast<uint4*>(wq + row * d + col);
        dst[0] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        dst[1] = make_uint4(wh[4], wh[5], wh[6], wh[7]);
      }
      if (active && (tx & (gthreads - 1)) == 0) {
        if (codes != nullptr) {
          scales[row * ngroups + kgroup] = s16;
          zeros[row * ngroups + kgroup] = __ushort_as_half(0);
        }
        ovf |= static_cast<bool>(__hisinf(s16)) || s * 448.0f > 65504.f;
      }
    }
  };
  int64_t base = static_cast<int64_t>(blockIdx.y) * rpi;
  for (; base < dp; base += 2 * stride) {
    if (base + stride < dp) load_rows(base + stride, nxt);
    process(base, cur);
    if (base + stride >= dp) break;
    if (base + 2 * stride < dp) load_rows(base + 2 * stride, cur);
    process(base + stride, nxt);
  }
  if (__any_sync(0xffffffffu, ovf) && lane == 0)
    set_flag(status, TTQ_FLAG_NONFINITE | TTQ_FLAG_SCALE_OVERFLOW);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_flag(status, TTQ_FLAG_NONFINITE);
}

// Largest tile width (a power of two in [32, 4096]) that divides d and is a
// multiple of the group.
int tile_width(int64_t d, int group) {
  for (int c = 4096; c >= 32; c >>= 1)
    if (c >= group && d % c == 0) return c;
  return group;
}

template <int BITS, bool WQ, bool SYM, int G>
cudaError_t launch_stage_g(dim3 grid, const __nv_bfloat16* W, int64_t dp, int64_t d,
                           const float* D, int cw, uint32_t* codes, __half* s, __half* z,
                           __half* wq, uint32_t* status, cudaStream_t stream, bool pdl) {
  constexpr size_t smem = kQSmemBytes;
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e = cudaFuncSetAttribute(qdq_stage_kernel<BITS, WQ, SYM, G>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_relaxed);
  }
  // narrow tiles (at most 256 channels, a batch of at most 256 rows): each
  // batch comes in as one tensor-map box instead of one bulk copy per row
  CUtensorMap tmW;
  memset(&tmW, 0, sizeof(tmW));
  const int rows_pb = kStageRows * (kThreads / (cw >> 4));
  const int w_box = cw <= 256 && rows_pb <= 256 && encode_bf16_box(&tmW, W, d, dp, cw, rows_pb);
  return launch_kernel(qdq_stage_kernel<BITS, WQ, SYM, G>, grid, dim3(kThreads), smem, stream,
                       pdl, tmW, w_box, W, dp, d, D, cw, codes, s, z, wq, status);
}

template <int BITS, bool WQ, bool SYM>
cudaError_t launch_stage(dim3 grid, const __nv_bfloat16* W, int64_t dp, int64_t d,
                         const float* D, int group, int cw, uint32_t* codes, __half* s,
                         __half* z, __half* wq, uint32_t* status, cudaStream_t stream, bool pdl) {
  switch (group) {
    case 32:
      return launch_stage_g<BITS, WQ, SYM, 2>(grid, W, dp, d, D, cw, codes, s, z, wq, status,
                                              stream, pdl);
    case 64:
      return launch_stage_g<BITS, WQ, SYM, 4>(grid, W, dp, d, D, cw, codes, s, z, wq, status,
                                              stream, pdl);
    case 128:
      return launch_stage_g<BITS, WQ, SYM, 8>(grid, W, dp, d, D, cw, codes, s, z, wq, status,
                                              stream, pdl);
    case 256:
      return launch_stage_g<BITS, WQ, SYM, 16>(grid, W, dp, d, D, cw, codes, s, z, wq, status,
                                               stream, pdl);
    default:
      return cudaErrorInvalidValue;
  }
}

// The launch of the staged kernel for bf16 W: one block per tile of cw
// channels and per gy row-batch slot, about two resident blocks per SM.
template <bool WQ, bool SYM>
cudaError_t launch_staged(const __nv_bfloat16* W, int64_t dp, int64_t d, const float* D,
                          int bits, int group, uint32_t* codes, uint16_t* scales,
                          uint16_t* zeros, void* wq, uint32_t* status, int num_sms,
                          cudaStream_t stream, bool pdl) {
  const int cw = tile_width(d, group);
  const int rows_pb = kStageRows * (kThreads / (cw >> 4));
  const int64_t gx = d / cw;
  const int64_t nb_all = (dp + rows_pb - 1) / rows_pb;
  // two resident blocks per SM, all in one wave
  int64_t gy = static_cast<int64_t>(num_sms) * 2 / gx;
  if (gy > nb_all) gy = nb_all;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  __half* s = reinterpret_cast<__half*>(scales);
  __half* z = reinterpret_cast<__half*>(zeros);
  __half* w = static_cast<__half*>(wq);
  switch (bits) {
    case 2:
      return launch_stage<2, WQ, SYM>(grid, W, dp, d, D, group, cw, codes, s, z, w, status,
                                      stream, pdl);
    case 3:
      return launch_stage<3, WQ, SYM>(grid, W, dp, d, D, group, cw, codes, s, z, w, status,
                                      stream, pdl);
    case 4:
      return launch_stage<4, WQ, SYM>(grid, W, dp, d, D, group, cw, codes, s, z, w, status,
                                      stream, pdl);
    default:
      return cudaErrorInvalidValue;
  }
}

template <typename WT, bool WQ, bool SYM>
cudaError_t launch_w(const WT* W, int64_t dp, int64_t d, const float* D, int bits, int group,
                     uint32_t* codes, uint16_t* scales, uint16_t* zeros, void* wq,
                     uint32_t* status, int num_sms, cudaStream_t stream, bool pdl) {
  const int cw = tile_width(d, group);
  const int rpi = kThreads / (cw >> 4);
  const int64_t gx = d / cw;
  const int64_t want = static_cast<int64_t>(num_sms) * 2;  // two resident blocks per SM
  int64_t gy = want / gx;   // all blocks resident in one wave
  const int64_t max_gy = (dp + rpi - 1) / rpi;  // each block still takes >= 1 row
  if (gy > max_gy) gy = max_gy;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  __half* s = reinterpret_cast<__half*>(scales);
  __half* z = reinterpret_cast<__half*>(zeros);
  switch (bits) {
    case 2:
      return launch_kernel(qdq_pack_kernel<WT, 2, WQ, SYM>, grid, dim3(kThreads), 0, stream, pdl, W, dp,
                           d, D, group, cw, codes, s, z, static_cast<__half*>(wq), status);
    case 3:
      return launch_kernel(qdq_pack_kernel<WT, 3, WQ, SYM>, grid, dim3(kThreads), 0, stream, pdl, W, dp,
                           d, D, group, cw, codes, s, z, static_cast<__half*>(wq), status);
    case 4:
      return launch_kernel(qdq_pack_kernel<WT, 4, WQ, SYM>, grid, dim3(kThreads), 0, stream, pdl, W, dp,
                           d, D, group, cw, codes, s, z, static_cast<__half*>(wq), status);
    default:
      return cudaErrorInvalidValue;
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               int64_t n8) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 2 * i + 1);
    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<uint4*>(h);
  }
}

// X' = binary16(X[t][i] * Dr[i]) (Dr == null: plain conversion).  A thread
// owns 8 consecutive channels (blockIdx.x, threadIdx.x) and walks the tokens
// with a grid stride, so its 8 factors are loaded once; flags X_RANGE if
// some |X'| > 65504.
template <typename T>
__global__ void __launch_bounds__(256) scale_to_f16_kernel(const T* __restrict__ src,
                                                           const float* __restrict__ Dr,
                                                           __half* __restrict__ dst, int64_t T_,
                                                           int64_t d, uint32_t* __restrict__ status) {
  const int64_t col = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) * 8;
  bool out_of_range = false;
  allow_dependents_launch();
  grid_dependency_wait();  // Dr comes from the previous kernel
  if (col < d) {
    float f[8];
    if (Dr != nullptr) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(Dr + col));
      const float4 b = __ldg(reinterpret_cast<const float4*>(Dr + col) + 1);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = 1.0f;
    }
    constexpr int kRows = 4;  // rows loaded before any is converted
    for (int64_t t0 = blockIdx.y; t0 < T_; t0 += static_cast<int64_t>(gridDim.y) * kRows) {
      uint4 raw[kRows][2];
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int64_t t = t0 + static_cast<int64_t>(u) * gridDim.y;
        if (t < T_) {
          const uint4* p = reinterpret_cast<const uint4*>(src + t * d + col);
          raw[u][0] = __ldcs(p);
          if constexpr (sizeof(T) == 4) raw[u][1] = __ldcs(p + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int64_t t = t0 + static_cast<int64_t>(u) * gridDim.y;
        if (t >= T_) continue;
        float v[8];
        if constexpr (sizeof(T) == 4) {
          v[0] = __uint_as_float(raw[u][0].x); v[1] = __uint_as_float(raw[u][0].y);
          v[2] = __uint_as_float(raw[u][0].z); v[3] = __uint_as_float(raw[u][0].w);
          v[4] = __uint_as_float(raw[u][1].x); v[5] = __uint_as_float(raw[u][1].y);
          v[6] = __uint_as_float(raw[u][1].z); v[7] = __uint_as_float(raw[u][1].w);
        } else if constexpr (std::is_same<T, __half>::value) {
          const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
            v[2 * k] = f2.x;
            v[2 * k + 1] = f2.y;
          }
        } else {
          const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(w[k] << 16);
            v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
          }
        }
        __half2 h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = v[2 * k] * f[2 * k];
          const float b = v[2 * k + 1] * f[2 * k + 1];
          h[k] = __floats2half2_rn(a, b);
          out_of_range |= !(fabsf(a) <= 65504.f) || !(fabsf(b) <= 65504.f);
        }
        *reinterpret_cast<uint4*>(dst + t * d + col) = *reinterpret_cast<uint4*>(h);
      }
    }
  }
  if (__any_sync(0xffffffffu, out_of_range) && (threadIdx.x & 31) == 0)
    set_flag(status, TTQ_FLAG_X_RANGE);
}

}  // namespace

cudaError_t launch_scale_to_f16(const void* src, int src_kind, const float* Dr, void* dst,
                                int64_t T, int64_t d, uint32_t* status, int num_sms,
                                cudaStream_t stream, bool pdl) {
  if (T == 0 || d == 0) return cudaSuccess;
  const int64_t gx = (d / 8 + 255) / 256;
  int64_t gy = (static_cast<int64_t>(num_sms) * 8 + gx - 1) / gx;
  if (gy > T) gy = T;
  if (gy > 65535) gy = 65535;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  __half* out = static_cast<__half*>(dst);
  if (src_kind == kSrcF32)
    return launch_kernel(scale_to_f16_kernel<float>, grid, dim3(256), 0, stream, pdl,
                         static_cast<const float*>(src), Dr, out, T, d, status);
  if (src_kind == kSrcF16)
    return launch_kernel(scale_to_f16_kernel<__half>, grid, dim3(256), 0, stream, pdl,
                         static_cast<const __half*>(src), Dr, out, T, d, status);
  return launch_kernel(scale_to_f16_kernel<__nv_bfloat16>, grid, dim3(256), 0, stream, pdl,
                       static_cast<const __nv_bfloat16*>(src), Dr, out, T, d, status);
}

template <typename WT, bool SYM>
cudaError_t launch_wq(const WT* W, int64_t dp, int64_t d, const float* D, int bits, int group,
                      uint32_t* codes, uint16_t* scales, uint16_t* zeros, void* wq,
                      uint32_t* status, int num_sms, cudaStream_t stream, bool pdl) {
  if constexpr (std::is_same<WT, __nv_bfloat16>::value) {
    // bf16 W: the kernel with W staged in shared memory
    return wq ? launch_staged<true, SYM>(W, dp, d, D, bits, group, codes, scales, zeros, wq,
                                         status, num_sms, stream, pdl)
              : launch_staged<false, SYM>(W, dp, d, D, bits, group, codes, scales, zeros, wq,
                                          status, num_sms, stream, pdl);
  } else {
    return wq ? launch_w<WT, true, SYM>(W, dp, d, D, bits, group, codes, scales, zeros, wq, status,
                                        num_sms, stream, pdl)
              : launch_w<WT, false, SYM>(W, dp, d, D, bits, group, codes, scales, zeros, wq,
                                         status, num_sms, stream, pdl);
  }
}

template <typename WT>
cudaError_t launch_scheme(const WT* W, int64_t dp, int64_t d, const float* D, int bits, int group,
                          bool symmetric, uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                          void* wq, uint32_t* status, int num_sms, cudaStream_t stream,
                          bool pdl) {
  return symmetric ? launch_wq<WT, true>(W, dp, d, D, bits, group, codes, scales, zeros, wq,
                                         status, num_sms, stream, pdl)
                   : launch_wq<WT, false>(W, dp, d, D, bits, group, codes, scales, zeros, wq,
                                          status, num_sms, stream, pdl);
}

cudaError_t launch_qdq_pack(const void* W, bool w_f32, int64_t dp, int64_t d, const float* D,
                            int bits, int group, uint32_t* codes, uint16_t* scales,
                            uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream, bool pdl, void* wq, bool symmetric) {
  if (dp == 0) return cudaSuccess;
  if (w_f32)
    return launch_scheme(static_cast<const float*>(W), dp, d, D, bits, group, symmetric, codes,
                         scales, zeros, wq, status, num_sms, stream, pdl);
  return launch_scheme(static_cast<const __nv_bfloat16*>(W), dp, d, D, bits, group, symmetric,
                       codes, scales, zeros, wq, status, num_sms, stream, pdl);
}

cudaError_t launch_qdq_fp8(const void* W, bool w_f32, int64_t dp, int64_t d, const float* D,
                           int group, uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                           uint32_t* status, int num_sms, cudaStream_t stream, bool pdl, void* wq) {
  if (dp == 0) return cudaSuccess;
  const int cw = tile_width(d, group);
  const int rpi = kThreads / (cw >> 4);
  const int64_t gx = d / cw;
  const int64_t want = static_cast<int64_t>(num_sms) * 2;
  int64_t gy = want / gx;   // all blocks resident in one wave
  const int64_t max_gy = (dp + rpi - 1) / rpi;
  if (gy > max_gy) gy = max_gy;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  __half* s = reinterpret_cast<__half*>(scales);
  __half* z = reinterpret_cast<__half*>(zeros);
  __half* w = static_cast<__half*>(wq);
  if (w_f32) {
    const float* Wf = static_cast<const float*>(W);
    return wq ? launch_kernel(qdq_fp8_kernel<float, true>, grid, dim3(kThreads), 0, stream, pdl, Wf, dp,
                              d, D, group, cw, codes, s, z, w, status)
              : launch_kernel(qdq_fp8_kernel<float, false>, grid, dim3(kThreads), 0, stream, pdl, Wf,
                              dp, d, D, group, cw, codes, s, z, w, status);
  }
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  return wq ? launch_kernel(qdq_fp8_kernel<__nv_bfloat16, true>, grid, dim3(kThreads), 0, stream, pdl,
                            Wb, dp, d, D, group, cw, codes, s, z, w, status)
            : launch_kernel(qdq_fp8_kernel<__nv_bfloat16, false>, grid, dim3(kThreads), 0, stream, pdl,
                            Wb, dp, d, D, group, cw, codes, s, z, w, status);
}

cudaError_t launch_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      src, static_cast<__nv_bfloat16*>(dst), n8);
  return cudaGetLastError();
}

}  // namespace ttq
