// Step (1) of the TTQ layer: the per-channel activation statistic
//   D_ii = (||X_i,:||_p + lambda)^alpha,  and D_ii^(-1/2)
// (gist.science/zh/paper/2603.19296, section 2.1).  X is [T][d] (token
// major), so channel i is a column: the reduction runs down the columns.
//
// The order of the sums, shared by both kernels below so that D is the same
// bits whichever runs: the tokens are cut into `splits` consecutive splits
// (act_norm_plan); within a split, |x|^p of channel i is accumulated in fp64
// over 16 row phases (phase j holds rows j, j + 16, j + 32, ... of the split,
// in increasing order), the 16 phase sums are added in phase order, and the
// split sums in split order.  fp64 is cheap here: the pass is bound by
// memory, not by the fp64 pipe.
//
// act_norm_kernel (any T): a block owns 256 consecutive channels and one
// split; lane l loads channels 8l..8l+7 of a row (one 16-byte load for
// bf16), warp w walks rows w, w + 8, ... of the split and so holds phases w
// and w + 8.  The split's sums go to global memory; the last block of a
// column block to finish (an atomic ticket) merges the splits.
//
// act_norm_scale_kernel (each split's rows fit in registers): the fused
// statistic and product operand X D^(-1/2), reading X from HBM once; the
// splits of a column block form one thread-block cluster and merge through
// distributed shared memory.
#include <map>
#include <mutex>
#include <utility>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kChannelsPerBlock = 256;  // act_norm_kernel's column block
constexpr int kClusterChannels = 128;   // act_norm_scale_kernel's column block
constexpr int kThreads = 256;
constexpr int kPhases = 16;             // row phases of a split
constexpr int kMaxSplits = 16;          // token splits (act_norm_plan)
constexpr int kMaxClusterSplits = 8;    // portable cluster size

// |x|^p in fp64: exact for p = 1 and for p = 2 with 16-bit inputs, so the
// merged sums (and hence D rounded to binary32) match an fp64 reference.
template <int PK>  // 1: p = 1, 2: p = 2, 0: any p >= 1
__device__ __forceinline__ double abs_pow(float x, double p) {
  const double a = fabs(static_cast<double>(x));
  if (PK == 1) return a;
  if (PK == 2) return a * a;
  return pow(a, p);
}

// D_ii and D_ii^(-1/2) (binary32) from the merged sum of |x|^p of channel
// i; false when either is zero, infinite or NaN.
template <int PK>
__device__ __forceinline__ bool finish_channel(double tot, double p, double lambda, double alpha,
                                               float* df, float* drf) {
  double n;
  if (PK == 1) {
    n = tot;
  } else if (PK == 2) {
    n = sqrt(tot);
  } else {
    n = pow(tot, 1.0 / p);
  }
  // (n + lambda)^alpha: the exponents the workloads use through correctly
  // rounded square roots (alpha = 1/2 is then the correctly rounded power
  // itself), any other through pow
  const double y = n + lambda;
  const double dv = alpha == 0.5   ? sqrt(y)
                    : alpha == 1.0  ? y
                    : alpha == 0.25 ? sqrt(sqrt(y))
                    : alpha == 0.0  ? 1.0
                                    : pow(y, alpha);
  const double drv = 1.0 / sqrt(dv);
  *df = static_cast<float>(dv);
  *drf = static_cast<float>(drv);
  return (*df > 0.f) && (*df <= 3.402823466e38f) && (*drf > 0.f) && (*drf <= 3.402823466e38f);
}

__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void load8(const float* src, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8_f16(__half* dst, const float (&v)[8]) {
  uint4 raw;
  __half2 h0 = __floats2half2_rn(v[0], v[1]);
  __half2 h1 = __floats2half2_rn(v[2], v[3]);
  __half2 h2 = __floats2half2_rn(v[4], v[5]);
  __half2 h3 = __floats2half2_rn(v[6], v[7]);
  raw.x = *reinterpret_cast<uint32_t*>(&h0);
  raw.y = *reinterpret_cast<uint32_t*>(&h1);
  raw.z = *reinterpret_cast<uint32_t*>(&h2);
  raw.w = *reinterpret_cast<uint32_t*>(&h3);
  *reinterpret_cast<uint4*>(dst) = raw;
}

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* dst, const float (&v)[8]) {
  uint4 raw;
  __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
  __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
  __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
  raw.x = *reinterpret_cast<uint32_t*>(&h0);
  raw.y = *reinterpret_cast<uint32_t*>(&h1);
  raw.z = *reinterpret_cast<uint32_t*>(&h2);
  raw.w = *reinterpret_cast<uint32_t*>(&h3);
  *reinterpret_cast<uint4*>(dst) = raw;
}

template <typename XT, int PK>
__global__ void __launch_bounds__(kThreads, 2) act_norm_kernel(
    const XT* __restrict__ X, int64_t d, int64_t T, double p, double lambda, double alpha,
    int64_t splits, int64_t rows_per_split, double* __restrict__ partial,
    uint32_t* __restrict__ counters, float* __restrict__ D, float* __restrict__ Dr,
    float* __restrict__ Dh, __half* __restrict__ xh, __nv_bfloat16* __restrict__ xb,
    uint32_t* __restrict__ status) {
  __shared__ double red[kPhases][kChannelsPerBlock + 2];
  __shared__ int is_last;
  allow_dependents_launch();
  grid_dependency_wait();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t cb = blockIdx.x;
  const int64_t sp = blockIdx.y;
  const int64_t c0 = cb * kChannelsPerBlock + lane * 8;

  // acc[h]: phase warp + 8h (rows warp + 8m of the split with m % 2 == h)
  double acc[2][8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[0][e] = acc[1][e] = 0.0;

  const int64_t t_begin = sp * rows_per_split;
  const int64_t t_end = min(T, t_begin + rows_per_split);
  float amax = 0.f;
  if (c0 < d) {
    // rows t_begin + warp + 8m, kBatch at a time (batches start at even m);
    // the next batch is loaded while the current one is summed.  A row past
    // the split is loaded as zeros and adds +0 to its phase, which leaves
    // the (non-negative or NaN) sum unchanged.
    constexpr int kBatch = 4;
    float v[kBatch][8], vn[kBatch][8];
    auto load_batch = [&](int64_t t0, float (&dst)[kBatch][8]) {
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int64_t t = t0 + 8 * k;
        if (t < t_end) {
          load8(X + t * d + c0, dst[k]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[k][e] = 0.f;
        }
      }
    };
    auto consume = [&](int64_t t0, const float(&buf)[kBatch][8]) {
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int64_t t = t0 + 8 * k;
        if (t < t_end) {
          if (xh != nullptr) store8_f16(xh + t * d + c0, buf[k]);
          if (xb != nullptr) store8_bf16(xb + t * d + c0, buf[k]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[k & 1][e] += abs_pow<PK>(buf[k][e], p);
          amax = fmaxf(amax, fabsf(buf[k][e]));
        }
      }
    };
    // ping-pong between two buffers (loop unrolled twice)
    constexpr int kStep = 8 * kBatch;
    int64_t t0 = t_begin + warp;
    if (t0 < t_end) load_batch(t0, v);
    for (; t0 < t_end; t0 += 2 * kStep) {
      if (t0 + kStep < t_end) load_batch(t0 + kStep, vn);
      consume(t0, v);
      if (t0 + kStep >= t_end) break;
      if (t0 + 2 * kStep < t_end) load_batch(t0 + 2 * kStep, v);
      consume(t0 + kStep, vn);
    }
  }
  // the binary16 copy of X holds |x| <= 65504 only (NaN is caught by D)
  if (xh != nullptr && __any_sync(0xffffffffu, amax > 65504.f) && lane == 0)
    set_flag(status, TTQ_FLAG_X_RANGE);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red[warp][lane * 8 + e] = acc[0][e];
    red[warp + 8][lane * 8 + e] = acc[1][e];
  }
  __syncthreads();

  const int ci = threadIdx.x;
  const int64_t c = cb * kChannelsPerBlock + ci;
  double sum = 0.0;
#pragma unroll
  for (int j = 0; j < kPhases; ++j) sum += red[j][ci];
  if (c < d) partial[sp * d + c] = sum;

  // Ticket: the last split block of this column block merges all splits.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&counters[cb], 1u);
    is_last = (prev == static_cast<uint32_t>(splits - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  if (c < d) {
    // split order; all partials loaded at once (one L2 round trip); the
    // +0 of an absent split leaves the sum unchanged
    double v[kMaxSplits];
#pragma unroll
    for (int k = 0; k < kMaxSplits; ++k) v[k] = k < splits ? __ldcg(partial + k * d + c) : 0.0;
    double tot = 0.0;
#pragma unroll
    for (int k = 0; k < kMaxSplits; ++k) tot += v[k];
    float df, drf;
    const bool ok = finish_channel<PK>(tot, p, lambda, alpha, &df, &drf);
    D[c] = df;
    Dr[c] = drf;
    if (Dh != nullptr) Dh[c] = __fsqrt_rn(df);   // the quantiser's h = sqrtf(D)
    if (!ok) set_flag(status, TTQ_FLAG_NONFINITE);
  }
  if (threadIdx.x == 0) counters[cb] = 0u;  // ready for the next call
}

// ---------------------------------------------------------------------------
// Fused form of the statistic pass and of the binary16 operand X D^(-1/2).
// Block (cb, sp) owns channels 128 cb .. 128 cb + 127 and split sp of the
// tokens.  Lane l of warp w takes channels 8 (l % 16) .. + 7 of the rows of
// phase j = 2w + l / 16 (rows j, j + 16, ... of the split), so a warp reads
// two whole 256-byte row segments per load.  Each thread loads all of its
// rows (at most reg_rows<XT>()) into registers at once, sums |x|^p over them
// in increasing row order, and the block adds its 16 phase sums in phase
// order.  The splits of a column block are the blocks of one thread-block
// cluster: each publishes its split sums in shared memory, and after the
// cluster barrier every block reads all of them through distributed shared
// memory and adds them in split order (the merge of act_norm_kernel, so D is
// identical).  It then writes binary16(x * D^(-1/2)) from the registers.  X
// is read from HBM once, and no block waits on another beyond its cluster,
// so no grid-wide residency is needed.

// Rows per thread held in registers: 16 uint4 of X.
template <typename XT>
__host__ __device__ constexpr int reg_rows() { return sizeof(XT) == 2 ? 16 : 8; }

template <typename XT>
struct Raw8;  // eight consecutive elements of X as loaded
template <>
struct Raw8<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16* src) {
    w = __ldcs(reinterpret_cast<const uint4*>(src));
  }
  __device__ __forceinline__ void unpack(float (&v)[8]) const {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* src) {
    a = __ldcs(reinterpret_cast<const float4*>(src));
    b = __ldcs(reinterpret_cast<const float4*>(src) + 1);
  }
  __device__ __forceinline__ void unpack(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

template <typename XT, int PK>
__global__ void __launch_bounds__(kThreads, 2) act_norm_scale_kernel(
    const XT* __restrict__ X, int64_t d, int64_t T, double p, double lambda, double alpha,
    int64_t splits, int64_t rows_per_split, float* __restrict__ D, float* __restrict__ Dr,
    float* __restrict__ Dh, __half* __restrict__ xh, __nv_bfloat16* __restrict__ xb,
    uint32_t* __restrict__ status) {
  constexpr int R = reg_rows<XT>();
  __shared__ double red[kPhases][kClusterChannels + 2];
  __shared__ double own_s[kClusterChannels];   // this split's sums, read by the cluster
  __shared__ float dr_s[kClusterChannels];
  allow_dependents_launch();
  grid_dependency_wait();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int phase = 2 * warp + (lane >> 4);
  const int cl = (lane & 15) * 8;
  const int64_t cb = blockIdx.x;
  const int64_t sp = blockIdx.y;   // also this block's rank in its cluster
  const int64_t c0 = cb * kClusterChannels + cl;
  const bool active = c0 < d;
  const int64_t t_begin = sp * rows_per_split;
  const int64_t t_end = min(T, t_begin + rows_per_split);
  const bool clustered = splits > 1;

  // this thread's rows: t0 + 16 k for k < nk (none when its channels are
  // past d), at a fixed stride from one base pointer
  const int64_t t0 = t_begin + phase;
  const int nk = active && t0 < t_end
                     ? static_cast<int>(min(static_cast<int64_t>(R), (t_end - t0 + kPhases - 1) / kPhases))
                     : 0;
  const int64_t rs = kPhases * d;
  const XT* xp = X + (nk > 0 ? t0 * d + c0 : 0);

  // all rows of this thread in flight at once
  Raw8<XT> raw[R];
#pragma unroll
  for (int k = 0; k < R; ++k)
    if (k < nk) raw[k].load(xp + k * rs);

  // (1) this phase's sums of |x|^p, rows in increasing order
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll
  for (int k = 0; k < R; ++k) {
    if (k < nk) {
      float v[8];
      raw[k].unpack(v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += abs_pow<PK>(v[e], p);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[phase][cl + e] = acc[e];
  __syncthreads();
  const int ci = threadIdx.x;   // channel of the merge, threads < 128
  const int64_t c = cb * kClusterChannels + ci;
  if (ci < kClusterChannels) {
    double own = 0.0;
#pragma unroll
    for (int j = 0; j < kPhases; ++j) own += red[j][ci];
    own_s[ci] = own;
  }

  // (2) every split of this column block has published; merge in split
  // order.  With one split the merge is that split's own sum (0 + v is v).
  if (clustered) {
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  float drf = 0.f;
  if (ci < kClusterChannels && c < d) {
    double tot = own_s[ci];
    if (clustered) {
      double v[kMaxClusterSplits];
#pragma unroll
      for (int k = 0; k < kMaxClusterSplits; ++k)
        v[k] = k < splits ? ld_cluster_f64(&own_s[ci], static_cast<uint32_t>(k)) : 0.0;
      tot = 0.0;
#pragma unroll
      for (int k = 0; k < kMaxClusterSplits; ++k) tot += v[k];
    }
    float df;
    const bool ok = finish_channel<PK>(tot, p, lambda, alpha, &df, &drf);
    if (sp == 0) {
      D[c] = df;
      Dr[c] = drf;
      if (Dh != nullptr) Dh[c] = __fsqrt_rn(df);   // the quantiser's h = sqrtf(D)
      if (!ok) set_flag(status, TTQ_FLAG_NONFINITE);
    }
  }
  if (ci < kClusterChannels) dr_s[ci] = drf;
  // this block has read the other blocks' sums (their shared memory must
  // stay until every block of the cluster is past this point)
  if (clustered) cluster_arrive_relaxed();
  __syncthreads();

  // (3) binary16(x * D^(-1/2)) (and the bf16 copy of a float32 X); the
  // products go through the packed f32x2 multiply (each lane rounded as
  // the scalar one), and their largest magnitude is checked once
  float amax = 0.f;
  if (nk > 0) {
    float2 f[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) f[q] = make_float2(dr_s[cl + 2 * q], dr_s[cl + 2 * q + 1]);
    __half* hp = xh + t0 * d + c0;
#pragma unroll
    for (int k = 0; k < R; ++k) {
      if (k < nk) {
        float v[8];
        raw[k].unpack(v);
        __half2 h[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 a = __fmul2_rn(make_float2(v[2 * q], v[2 * q + 1]), f[q]);
          h[q] = __floats2half2_rn(a.x, a.y);
          amax = fmaxf(amax, fmaxf(fabsf(a.x), fabsf(a.y)));
        }
        *reinterpret_cast<uint4*>(hp + k * rs) = *reinterpret_cast<const uint4*>(h);
        if (xb != nullptr) store8_bf16(xb + t0 * d + c0 + k * rs, v);
      }
    }
  }
  // |x D^(-1/2)| beyond binary16 (a NaN x makes D NaN, flagged there)
  if (__any_sync(0xffffffffu, amax > 65504.f) && lane == 0) set_flag(status, TTQ_FLAG_X_RANGE);
  if (clustered) cluster_wait_acquire();
}

template <typename XT, int PK>
cudaError_t launch_typed(const XT* X, int64_t d, int64_t T, float p, float lambda, float alpha,
                         int64_t splits, int64_t rows_per_split, double* partial,
                         uint32_t* counters, float* D, float* Dr, float* Dh, void* xh, void* xb,
                         uint32_t* status, cudaStream_t stream, bool pdl) {
  const dim3 grid(static_cast<unsigned>((d + kChannelsPerBlock - 1) / kChannelsPerBlock),
                  static_cast<unsigned>(splits));
  return launch_kernel(act_norm_kernel<XT, PK>, grid, dim3(kThreads), 0, stream, pdl, X, d, T,
                       static_cast<double>(p), static_cast<double>(lambda),
                       static_cast<double>(alpha), splits, rows_per_split, partial, counters, D,
                       Dr, Dh, static_cast<__half*>(xh), static_cast<__nv_bfloat16*>(xb), status);
}

template <typename XT>
cudaError_t launch_p(const XT* X, int64_t d, int64_t T, float p, float lambda, float alpha,
                     int64_t splits, int64_t rows_per_split, double* partial, uint32_t* counters,
                     float* D, float* Dr, float* Dh, void* xh, void* xb, uint32_t* status,
                     cudaStream_t stream, bool pdl) {
  if (p == 1.0f)
    return launch_typed<XT, 1>(X, d, T, p, lambda, alpha, splits, rows_per_split, partial,
                               counters, D, Dr, Dh, xh, xb, status, stream, pdl);
  if (p == 2.0f)
    return launch_typed<XT, 2>(X, d, T, p, lambda, alpha, splits, rows_per_split, partial,
                               counters, D, Dr, Dh, xh, xb, status, stream, pdl);
  return launch_typed<XT, 0>(X, d, T, p, lambda, alpha, splits, rows_per_split, partial,
                             counters, D, Dr, Dh, xh, xb, status, stream, pdl);
}

// Whether a cluster of `splits` blocks of the fused kernel can be resident
// on this device (false when the query fails), cached per device and size.
template <typename XT, int PK>
bool cluster_resident(int64_t splits) {
  static std::mutex mu;
  static int8_t cache[64][kMaxClusterSplits + 1] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  int8_t& known = cache[dev][splits];
  if (known == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, static_cast<unsigned>(splits));
    cfg.blockDim = dim3(kThreads);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e =
        cudaOccupancyMaxActiveClusters(&n, act_norm_scale_kernel<XT, PK>, &cfg);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    known = n > 0 ? 1 : -1;
  }
  return known > 0;
}

// Whether the fused kernel applies: every thread's rows fit in its
// registers and the splits of a column block form one cluster.
template <typename XT, int PK>
bool fused_fits(int64_t splits, int64_t rows_per_split) {
  if (rows_per_split > kPhases * reg_rows<XT>()) return false;
  if (splits < 1 || splits > kMaxClusterSplits) return false;
  return splits == 1 || cluster_resident<XT, PK>(splits);
}

template <typename XT>
bool fused_fits_p(float p, int64_t splits, int64_t rows_per_split) {
  if (p == 1.0f) return fused_fits<XT, 1>(splits, rows_per_split);
  if (p == 2.0f) return fused_fits<XT, 2>(splits, rows_per_split);
  return fused_fits<XT, 0>(splits, rows_per_split);
}

template <typename XT, int PK>
cudaError_t launch_fused_typed(const XT* X, int64_t d, int64_t T, float p, float lambda,
                               float alpha, int64_t splits, int64_t rows_per_split, float* D,
                               float* Dr, float* Dh, void* xh, void* xb, uint32_t* status,
                               cudaStream_t stream, bool* launched) {
  *launched = false;
  if (!fused_fits<XT, PK>(splits, rows_per_split)) return cudaSuccess;
  const int64_t ncb = (d + kClusterChannels - 1) / kClusterChannels;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ncb), static_cast<unsigned>(splits));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  // may overlap the previous kernel's tail (the kernel waits for it before
  // touching memory); the splits of a column block are one cluster
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = static_cast<unsigned>(splits);
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = splits > 1 ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, act_norm_scale_kernel<XT, PK>, X, d, T, static_cast<double>(p),
      static_cast<double>(lambda), static_cast<double>(alpha), splits, rows_per_split, D, Dr, Dh,
      static_cast<__half*>(xh), static_cast<__nv_bfloat16*>(xb), status);
  *launched = e == cudaSuccess;
  return e;
}

template <typename XT>
cudaError_t launch_fused_p(const XT* X, int64_t d, int64_t T, float p, float lambda, float alpha,
                           int64_t splits, int64_t rows_per_split, float* D, float* Dr, float* Dh,
                           void* xh, void* xb, uint32_t* status, cudaStream_t stream,
                           bool* launched) {
  if (p == 1.0f)
    return launch_fused_typed<XT, 1>(X, d, T, p, lambda, alpha, splits, rows_per_split, D, Dr,
                                     Dh, xh, xb, status, stream, launched);
  if (p == 2.0f)
    return launch_fused_typed<XT, 2>(X, d, T, p, lambda, alpha, splits, rows_per_split, D, Dr,
                                     Dh, xh, xb, status, stream, launched);
  return launch_fused_typed<XT, 0>(X, d, T, p, lambda, alpha, splits, rows_per_split, D, Dr, Dh,
                                   xh, xb, status, stream, launched);
}

__global__ void sqrt_f32_kernel(const float* __restrict__ D, float* __restrict__ h, int64_t d) {
  allow_dependents_launch();
  grid_dependency_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < d;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    h[i] = __fsqrt_rn(D[i]);
}

}  // namespace

cudaError_t launch_sqrt_f32(const float* D, float* h, int64_t d, cudaStream_t stream) {
  if (d == 0) return cudaSuccess;
  int64_t blocks = (d + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  return launch_kernel(sqrt_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                       false, D, h, d);
}

void act_norm_plan(int64_t d, int64_t T, int num_sms, int64_t* splits, int64_t* rows_per_split) {
  // When 8 splits of at most 256 rows cover T (the fused kernel's register
  // capacity for bf16 X), as many splits as keep the 128-channel blocks
  // within two per SM (one wave), but enough for the rows to fit, at most 8
  // (one cluster).  Otherwise as many as keep the 256-channel blocks within
  // two per SM, at most 16.  Always at most one split per 32 rows.
  const int64_t fit = (T + kPhases * 16 - 1) / (kPhases * 16);
  const int64_t target = static_cast<int64_t>(num_sms) * 2;
  int64_t s;
  if (fit <= kMaxClusterSplits) {
    const int64_t ncb = (d + kClusterChannels - 1) / kClusterChannels;
    s = target / ncb;
    if (s < fit) s = fit;
    if (s > kMaxClusterSplits) s = kMaxClusterSplits;
  } else {
    const int64_t ncb = (d + kChannelsPerBlock - 1) / kChannelsPerBlock;
    s = target / ncb;
    if (s > kMaxSplits) s = kMaxSplits;
  }
  const int64_t max_by_rows = (T + 31) / 32;
  if (s > max_by_rows) s = max_by_rows;
  if (s < 1) s = 1;
  int64_t rps = (T + s - 1) / s;
  if (rps < 1) rps = 1;
  s = (T + rps - 1) / rps;
  if (s < 1) s = 1;
  *splits = s;
  *rows_per_split = rps;
}

cudaError_t launch_act_norm(const void* X, bool x_f32, int64_t d, int64_t T, float p,
                            float lambda, float alpha, int64_t splits, int64_t rows_per_split,
                            double* partial, uint32_t* counters, float* D, float* Dr, void* xh,
                            void* xb, uint32_t* status, cudaStream_t stream, bool pdl, float* Dh) {
  if (x_f32)
    return launch_p(static_cast<const float*>(X), d, T, p, lambda, alpha, splits, rows_per_split,
                    partial, counters, D, Dr, Dh, xh, xb, status, stream, pdl);
  return launch_p(static_cast<const __nv_bfloat16*>(X), d, T, p, lambda, alpha, splits,
                  rows_per_split, partial, counters, D, Dr, Dh, xh, nullptr, status, stream, pdl);
}

bool act_norm_scale_fused(bool x_f32, int64_t splits, int64_t rows_per_split, float p) {
  return x_f32 ? fused_fits_p<float>(p, splits, rows_per_split)
               : fused_fits_p<__nv_bfloat16>(p, splits, rows_per_split);
}

cudaError_t launch_act_norm_scale(const void* X, bool x_f32, int64_t d, int64_t T, float p,
                                  float lambda, float alpha, int64_t splits,
                                  int64_t rows_per_split, float* D, float* Dr, void* xh, void* xb,
                                  uint32_t* status, cudaStream_t stream, bool* launched,
                                  float* Dh) {
  if (x_f32)
    return launch_fused_p(static_cast<const float*>(X), d, T, p, lambda, alpha, splits,
                          rows_per_split, D, Dr, Dh, xh, xb, status, stream, launched);
  return launch_fused_p(static_cast<const __nv_bfloat16*>(X), d, T, p, lambda, alpha, splits,
                        rows_per_split, D, Dr, Dh, xh, nullptr, status, stream, launched);
}

}  // namespace ttq
