// Step (2) of the TTQ layer without the final rescale: codes, scales and
// zeros of Q[W D^{1/2}] (gist.science/zh/paper/2603.19296, section 2.1),
// with Q the group-wise asymmetric scale + zero-point quantiser (blog.lo0.es
// "Test-time quantization ...", section "The maths that matter").
//
// The arithmetic follows one fixed binary32 order so that the codes match
// the CPU oracle bit for bit:
//   h = sqrt(D_i); x = W_ji * h; m = min(0, min x); M = max(0, max x);
//   s32 = (M - m) / (2^b - 1), floored at 2^-14; s = binary16 round-up(s32);
//   inv = 1 / s; z = clamp(rint(-m * inv)); q = clamp(rint(x * inv) + z).
// Every operation is an explicitly rounded intrinsic, so no FMA contraction
// can change a result.
//
// Layout of the work: a block owns a tile of `cw` consecutive input channels
// and walks rows of W with a grid stride.  A thread owns 8 consecutive
// channels (one 16-byte load of bf16 W), keeps their sqrt(D) in registers
// for every row it visits, and the group's g/8 threads reduce min/max with
// shuffles.  Codes are assembled into 32-bit words across the 4 lanes that
// hold 32 consecutive codes (b words per 32 codes) and stored directly.
// The kernel is HBM-bound: it reads W once and writes d*b/8 + 4d/g bytes per
// row.
#include <type_traits>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void load8(const float* src, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(src));
  const float4 b = __ldcs(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename WT, int BITS>
__global__ void __launch_bounds__(kThreads) qdq_pack_kernel(
    const WT* __restrict__ W, int64_t dp, int64_t d, const float* __restrict__ D, int group,
    int cw, uint32_t* __restrict__ codes, __half* __restrict__ scales,
    __half* __restrict__ zeros, uint32_t* __restrict__ status) {
  constexpr int QMAX = (1 << BITS) - 1;
  const int tpr = cw >> 3;            // threads per row of the tile
  const int rpi = kThreads / tpr;     // rows per iteration of the block
  const int tx = threadIdx.x % tpr;
  const int ty = threadIdx.x / tpr;
  const int lane = threadIdx.x & 31;
  const int gthreads = group >> 3;    // threads sharing one group (4..32)
  const int64_t col = static_cast<int64_t>(blockIdx.x) * cw + tx * 8;
  const int64_t ngroups = d / group;
  const int64_t kgroup = col / group;  // this thread's group within the row
  const int64_t wpr = d * BITS / 32;  // words per row

  float h[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) h[e] = (D != nullptr) ? __fsqrt_rn(__ldg(D + col + e)) : 1.0f;
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) bad |= !(h[e] <= 3.402823466e38f);

  bool ovf = false;
  // The loop bound is block-uniform so every lane takes part in the
  // shuffles; rows past the end are computed on zeros and not stored.  Each
  // iteration issues the loads of kRows rows before using any of them.
  constexpr int kRows = 4;
  const int64_t step = static_cast<int64_t>(gridDim.y) * rpi;
  for (int64_t base = static_cast<int64_t>(blockIdx.y) * rpi; base < dp; base += kRows * step) {
    float x[kRows][8];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int64_t row = base + u * step + ty;
      if (row < dp) {
        load8(W + row * d + col, x[u]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int64_t row = base + u * step + ty;
      const bool active = row < dp;
      float mn = 0.f, mx = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[u][e] = __fmul_rn(x[u][e], h[e]);
        bad |= !(fabsf(x[u][e]) <= 3.402823466e38f);
        mn = fminf(mn, x[u][e]);
        mx = fmaxf(mx, x[u][e]);
      }
      for (int o = gthreads >> 1; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      float s32 = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(QMAX));
      if (!(s32 >= 6.103515625e-05f)) s32 = 6.103515625e-05f;  // 2^-14
      const __half s16 = __float2half_ru(s32);
      const float s = __half2float(s16);
      const float inv = __fdiv_rn(1.0f, s);
      const float zr = rintf(__fmul_rn(-mn, inv));
      const int z = static_cast<int>(fminf(fmaxf(zr, 0.f), static_cast<float>(QMAX)));
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int q = __float2int_rn(__fmul_rn(x[u][e], inv)) + z;
        q = min(max(q, 0), QMAX);
        packed |= static_cast<uint32_t>(q) << (BITS * e);
      }
      if (active && (tx & (gthreads - 1)) == 0) {
        scales[row * ngroups + kgroup] = s16;
        zeros[row * ngroups + kgroup] = __int2half_rn(z);
        // s (q - z) is formed in binary16 by the product: |q - z| <= 2^b - 1
        ovf |= static_cast<bool>(__hisinf(s16)) || s * static_cast<float>(QMAX) > 65504.f;
      }
      // 4 lanes hold 32 codes = BITS words; lane i of the quad writes word i.
      const int qbase = lane & ~3;
      const uint32_t v0 = __shfl_sync(0xffffffffu, packed, qbase + 0);
      const uint32_t v1 = __shfl_sync(0xffffffffu, packed, qbase + 1);
      const uint32_t v2 = __shfl_sync(0xffffffffu, packed, qbase + 2);
      const uint32_t v3 = __shfl_sync(0xffffffffu, packed, qbase + 3);
      const int qi = lane & 3;
      if (active && qi < BITS) {
        const unsigned __int128 stream =
            static_cast<unsigned __int128>(v0) | (static_cast<unsigned __int128>(v1) << (8 * BITS)) |
            (static_cast<unsigned __int128>(v2) << (16 * BITS)) |
            (static_cast<unsigned __int128>(v3) << (24 * BITS));
        const uint32_t word = static_cast<uint32_t>(stream >> (32 * qi));
        const int64_t quad_col = col - (tx & 3) * 8;  // first channel of the quad
        codes[row * wpr + (quad_col >> 5) * BITS + qi] = word;
      }
    }
  }
  if (__any_sync(0xffffffffu, ovf) && lane == 0)
    set_flag(status, TTQ_FLAG_NONFINITE | TTQ_FLAG_SCALE_OVERFLOW);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_flag(status, TTQ_FLAG_NONFINITE);
}

// Largest tile width (a power of two in [32, 2048]) that divides d and is a
// multiple of the group.
int tile_width(int64_t d, int group) {
  for (int c = 2048; c >= 32; c >>= 1)
    if (c >= group && d % c == 0) return c;
  return group;
}

template <typename WT>
cudaError_t launch_w(const WT* W, int64_t dp, int64_t d, const float* D, int bits, int group,
                     uint32_t* codes, uint16_t* scales, uint16_t* zeros, uint32_t* status,
                     int num_sms, cudaStream_t stream) {
  const int cw = tile_width(d, group);
  const int rpi = kThreads / (cw >> 3);
  const int64_t gx = d / cw;
  const int64_t want = static_cast<int64_t>(num_sms) * 8;
  int64_t gy = (want + gx - 1) / gx;
  const int64_t max_gy = (dp + rpi - 1) / rpi;  // each block still takes >= 1 row
  if (gy > max_gy) gy = max_gy;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  __half* s = reinterpret_cast<__half*>(scales);
  __half* z = reinterpret_cast<__half*>(zeros);
  switch (bits) {
    case 2:
      qdq_pack_kernel<WT, 2><<<grid, kThreads, 0, stream>>>(W, dp, d, D, group, cw, codes, s, z, status);
      break;
    case 3:
      qdq_pack_kernel<WT, 3><<<grid, kThreads, 0, stream>>>(W, dp, d, D, group, cw, codes, s, z, status);
      break;
    case 4:
      qdq_pack_kernel<WT, 4><<<grid, kThreads, 0, stream>>>(W, dp, d, D, group, cw, codes, s, z, status);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
    for (int64_t t = blockIdx.y; t < T_; t += gridDim.y) {
      float v[8];
      if constexpr (sizeof(T) == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(src + t * d + col));
        const float4 b = __ldg(reinterpret_cast<const float4*>(src + t * d + col) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else if constexpr (std::is_same<T, __half>::value) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + t * d + col));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
          v[2 * k] = f2.x;
          v[2 * k + 1] = f2.y;
        }
      } else {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + t * d + col));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
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
  if (__any_sync(0xffffffffu, out_of_range) && (threadIdx.x & 31) == 0)
    set_flag(status, TTQ_FLAG_X_RANGE);
}

}  // namespace

cudaError_t launch_scale_to_f16(const void* src, int src_kind, const float* Dr, void* dst,
                                int64_t T, int64_t d, uint32_t* status, int num_sms,
                                cudaStream_t stream) {
  if (T == 0 || d == 0) return cudaSuccess;
  const int64_t gx = (d / 8 + 255) / 256;
  int64_t gy = (static_cast<int64_t>(num_sms) * 8 + gx - 1) / gx;
  if (gy > T) gy = T;
  if (gy > 65535) gy = 65535;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  if (src_kind == kSrcF32)
    scale_to_f16_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(src), Dr,
                                                         static_cast<__half*>(dst), T, d, status);
  else if (src_kind == kSrcF16)
    scale_to_f16_kernel<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(src), Dr,
                                                          static_cast<__half*>(dst), T, d, status);
  else
    scale_to_f16_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(src), Dr, static_cast<__half*>(dst), T, d, status);
  return cudaGetLastError();
}

cudaError_t launch_qdq_pack(const void* W, bool w_f32, int64_t dp, int64_t d, const float* D,
                            int bits, int group, uint32_t* codes, uint16_t* scales,
                            uint16_t* zeros, uint32_t* status, int num_sms,
                            cudaStream_t stream) {
  if (dp == 0) return cudaSuccess;
  if (w_f32)
    return launch_w(static_cast<const float*>(W), dp, d, D, bits, group, codes, scales, zeros,
                    status, num_sms, stream);
  return launch_w(static_cast<const __nv_bfloat16*>(W), dp, d, D, bits, group, codes, scales,
                  zeros, status, num_sms, stream);
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
