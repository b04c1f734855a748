// Static low-rank initialisation of the TTQ layer: B, A from a truncated
// SVD of W, and the residual W - B A that the forward quantises
// (gist.science/zh/paper/2603.19296, section 2.2: W ~ W_q + B A with static
// B, A initialised by PCA; gist.science/nl/paper/2603.19296, section 2
// "Kerncomponenten", item 3).  PCA of W is read as W's uncentred truncated
// SVD, B = U_r S_r (d' x r), A = V_r^T (r x d).
//
// The SVD is a randomised range finder with subspace iteration (Halko,
// Martinsson and Tropp, "Finding structure with randomness", SIAM Review
// 2011, algorithms 4.4 and 5.1), all on the GPU:
//   Y = W Omega (Omega: the caller's d x l Gaussian test matrix, l = r + p)
//   Q = orth(Y); q times: Q = orth(W orth(W^T Q))
//   Bt = W^T Q (= (Q^T W)^T, d x l);  Bt^T Bt = U~ L U~^T (Jacobi, fp64)
//   sigma = sqrt(L); B = Q U~_r diag(sigma_r); A = diag(1 / sigma_r) U~_r^T Bt^T
//   W_res = W - B A (with B, A as stored)
// orth() is shifted CholeskyQR3: G = Y^T Y, G + shift I = R^T R,
// Y <- Y R^-1, three times, the first with shift = 1e-6 trace(G) (so that
// the fp32 Gram matrix of an ill-conditioned Y still factors) and the other
// two without.  R is invertible, so every pass keeps the span of Y; the
// shift only delays orthonormality to the later passes.
//
// The products are tall and skinny (l <= 96 columns) and W dominates their
// bytes; they run as fp32 CUDA-core GEMMs over strided operand views (no
// operand is transposed in memory), so the subspace keeps fp32 precision
// where binary16 or bf16 tensor-core operands would cost three to four
// decimal digits of the singular vectors.  Reductions over the long
// dimension split over CTAs into fp32 partial sums that a second kernel adds
// in split order in fp64 (deterministic).  The l x l factorisations run in
// one CTA in fp64 in shared memory.
#include <algorithm>
#include <type_traits>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kTM = 64, kTN = 64, kTK = 16, kGemmThreads = 256;

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
  if constexpr (std::is_same<T, float>::value) return __ldg(p);
  else return __bfloat162float(*p);
}

// Strided views and the epilogue of one product C = A B (M x N, reduction
// K): A(m, k) = A[m sam + k sak], B(k, n) = B[k sbk + n sbn].
struct GemmView {
  int64_t M, N, K;
  int64_t sam, sak, sbk, sbn;
  int splits;            // CTAs along K; > 1 writes fp32 partial sums
  int64_t kps;           // K per split
  float* partial;        // [splits][M][N] when splits > 1
  // epilogue (splits == 1 here, or in the finishing kernel):
  //   v = acc * col_scale[n] (if given);  v = sub(m, n) - v (if given)
  const float* col_scale;
  const void* sub;
  int sub_bf16;
  int64_t ssm, ssn;
  void* out;
  int out_type;          // 0 float, 1 bf16, 2 double
  int64_t som, son;
};

__device__ __forceinline__ void epilogue(const GemmView& g, int64_t m, int64_t n, double acc) {
  double v = acc;
  if (g.col_scale) v *= static_cast<double>(g.col_scale[n]);
  if (g.sub) {
    const int64_t at = m * g.ssm + n * g.ssn;
    const double w = g.sub_bf16 ? static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(g.sub)[at]))
                                : static_cast<double>(static_cast<const float*>(g.sub)[at]);
    v = w - v;
  }
  const int64_t at = m * g.som + n * g.son;
  if (g.out_type == 2) static_cast<double*>(g.out)[at] = v;
  else if (g.out_type == 1) static_cast<__nv_bfloat16*>(g.out)[at] = __float2bfloat16_rn(static_cast<float>(v));
  else static_cast<float*>(g.out)[at] = static_cast<float>(v);
}

// 64 x 64 tile per CTA, 4 x 4 outputs per thread, K in chunks of 16 staged
// in shared memory; each operand is loaded along whichever of its strides
// is 1 (coalesced), whatever the view's orientation.
template <typename TA, typename TB>
__global__ void __launch_bounds__(kGemmThreads) strided_gemm_kernel(GemmView g, const TA* __restrict__ A,
                                                                    const TB* __restrict__ B) {
  __shared__ __align__(16) float As[kTK][kTM];
  __shared__ __align__(16) float Bs[kTK][kTN];
  const int t = threadIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTN;
  const int64_t kb = static_cast<int64_t>(blockIdx.z) * g.kps;
  const int64_t ke = kb + g.kps < g.K ? kb + g.kps : g.K;
  const int tm = t / 16, tn = t % 16;
  const bool a_mfast = g.sam == 1;
  const bool b_nfast = g.sbn == 1;
  float acc[4][4] = {};
  // the next chunk's operands are loaded into registers while this one is
  // multiplied out of shared memory
  float ra[4], rb[4];
  auto load = [&](int64_t k0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = t + kGemmThreads * j;     // 0..1023
      const int mm = a_mfast ? (e % kTM) : (e / kTK);
      const int kk = a_mfast ? (e / kTM) : (e % kTK);
      const int64_t m = m0 + mm, k = k0 + kk;
      ra[j] = (m < g.M && k < ke) ? ldf(A + m * g.sam + k * g.sak) : 0.f;
      const int nn = b_nfast ? (e % kTN) : (e / kTK);
      const int kk2 = b_nfast ? (e / kTN) : (e % kTK);
      const int64_t n = n0 + nn, k2 = k0 + kk2;
      rb[j] = (n < g.N && k2 < ke) ? ldf(B + k2 * g.sbk + n * g.sbn) : 0.f;
    }
  };
  if (kb < ke) load(kb);
  for (int64_t k0 = kb; k0 < ke; k0 += kTK) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = t + kGemmThreads * j;
      As[a_mfast ? (e / kTM) : (e % kTK)][a_mfast ? (e % kTM) : (e / kTK)] = ra[j];
      Bs[b_nfast ? (e / kTN) : (e % kTK)][b_nfast ? (e % kTN) : (e / kTK)] = rb[j];
    }
    __syncthreads();
    if (k0 + kTK < ke) load(k0 + kTK);
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][tm * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tn * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + tm * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tn * 4 + j;
      if (n >= g.N) continue;
      if (g.splits > 1) g.partial[(static_cast<int64_t>(blockIdx.z) * g.M + m) * g.N + n] = acc[i][j];
      else epilogue(g, m, n, static_cast<double>(acc[i][j]));
    }
  }
}

// Adds the partial sums of a split product in split order (fp64) and
// applies the epilogue.
__global__ void finish_split_kernel(GemmView g) {
  const int64_t mn = g.M * g.N;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < mn;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int z = 0; z < g.splits; ++z) s += static_cast<double>(g.partial[z * mn + e]);
    epilogue(g, e / g.N, e % g.N, s);
  }
}

// Cholesky G + shift I = R^T R (R upper; shift = shift_rel trace(G)) of the
// l x l Gram matrix in fp64 and the upper-triangular inverse Rinv = R^-1
// (fp32 out).  A pivot that is not positive (fewer than l independent
// directions) is floored at max(1e-30 times the largest diagonal element,
// 1e-30) and flagged; the floor keeps R^-1 finite in fp32.
__global__ void chol_rinv_kernel(const double* __restrict__ G, int l, double shift_rel,
                                 float* __restrict__ Rinv, uint32_t* status) {
  extern __shared__ double sm[];
  double* R = sm;               // [l][l], upper triangle used
  double* X = sm + l * l;       // [l][l], the inverse
  const int t = threadIdx.x, nt = blockDim.x;
  for (int e = t; e < l * l; e += nt) {
    R[e] = G[e];
    X[e] = 0.0;
  }
  __syncthreads();
  __shared__ double dmax;
  if (t == 0) {
    double mx = 0.0, tr = 0.0;
    for (int i = 0; i < l; ++i) {
      mx = fmax(mx, R[i * l + i]);
      tr += R[i * l + i];
    }
    const double sh = shift_rel * tr;
    for (int i = 0; i < l; ++i) R[i * l + i] += sh;
    dmax = mx + sh;
  }
  __syncthreads();
  // right-looking: after column j is final, update the trailing block
  for (int j = 0; j < l; ++j) {
    if (t == 0) {
      double p = R[j * l + j];
      if (!(p > 1e-30 * dmax) || !(p > 1e-30)) {
        set_flag(status, TTQ_FLAG_RANK_DEFICIENT);
        p = fmax(1e-30 * dmax, 1e-30);
      }
      R[j * l + j] = sqrt(p);
    }
    __syncthreads();
    const double rjj = R[j * l + j];
    for (int i = j + 1 + t; i < l; i += nt) R[j * l + i] /= rjj;
    __syncthreads();
    // G[a][b] -= R[j][a] R[j][b] for j < a <= b
    for (int e = t; e < (l - j - 1) * (l - j - 1); e += nt) {
      const int a = j + 1 + e / (l - j - 1), b = j + 1 + e % (l - j - 1);
      if (b >= a) R[a * l + b] -= R[j * l + a] * R[j * l + b];
    }
    __syncthreads();
  }
  // R X = I by back substitution, one column per thread
  for (int c = t; c < l; c += nt) {
    X[c * l + c] = 1.0 / R[c * l + c];
    for (int i = c - 1; i >= 0; --i) {
      double s = 0.0;
      for (int k = i + 1; k <= c; ++k) s += R[i * l + k] * X[k * l + c];
      X[i * l + c] = -s / R[i * l + i];
    }
  }
  __syncthreads();
  for (int e = t; e < l * l; e += nt) {
    const double v = X[e];
    if (!isfinite(v)) set_flag(status, TTQ_FLAG_NONFINITE);
    Rinv[e] = static_cast<float>(v);
  }
}

// Symmetric eigendecomposition of the l x l matrix S (fp64) by cyclic
// Jacobi rotations in round-robin order (l/2 disjoint planes per round, all
// rotated at once), at most 40 sweeps or until the off-diagonal mass falls
// below 1e-28 of the total.  Out: eigenvectors as columns of U (fp32),
// sorted by descending eigenvalue, sigma = sqrt(max(eigenvalue, 0)) and
// 1 / sigma, taken as 0 where sigma <= 1e-6 sigma_max (such a direction is
// dropped from A: its column of B is at most 1e-6 sigma_max anyway).
__global__ void jacobi_eig_kernel(const double* __restrict__ S, int l, float* __restrict__ U,
                                  float* __restrict__ sigma, float* __restrict__ inv_sigma,
                                  uint32_t* status) {
  extern __shared__ double sm[];
  const int n = (l + 1) & ~1;   // even number of slots (one dummy when l is odd)
  double* G = sm;               // [l][l]
  double* V = G + l * l;        // [l][l]
  double* cs = V + l * l;       // [n/2] cos
  double* sn = cs + n / 2;      // [n/2] sin
  int* pp = reinterpret_cast<int*>(sn + n / 2);
  int* qq = pp + n / 2;
  int* order = qq + n / 2;      // [l]
  __shared__ double red[32];
  __shared__ int done;
  const int t = threadIdx.x, nt = blockDim.x;
  for (int e = t; e < l * l; e += nt) {
    G[e] = S[e];
    V[e] = (e / l == e % l) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < 40; ++sweep) {
    // convergence: off-diagonal against total squared mass
    double off = 0.0, tot = 0.0;
    for (int e = t; e < l * l; e += nt) {
      const double v = G[e] * G[e];
      tot += v;
      if (e / l != e % l) off += v;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((t & 31) == 0) {
      red[t >> 5] = off;
      red[16 + (t >> 5)] = tot;
    }
    __syncthreads();
    if (t == 0) {
      double o2 = 0.0, t2 = 0.0;
      for (int w = 0; w < (nt + 31) / 32; ++w) {
        o2 += red[w];
        t2 += red[16 + w];
      }
      done = !(o2 > 1e-28 * t2);
    }
    __syncthreads();
    if (done) break;
    for (int round = 0; round < n - 1; ++round) {
      // slot 0 stays, slots 1..n-1 rotate; pair i is (slot i, slot n-1-i)
      for (int i = t; i < n / 2; i += nt) {
        auto slot = [&](int s) { return s == 0 ? 0 : 1 + (s - 1 + round) % (n - 1); };
        int p = slot(i), q = slot(n - 1 - i);
        if (p > q) {
          const int x = p;
          p = q;
          q = x;
        }
        double c = 1.0, s = 0.0;
        if (q < l) {
          const double apq = G[p * l + q];
          if (apq != 0.0) {
            const double theta = (G[q * l + q] - G[p * l + p]) / (2.0 * apq);
            const double tt = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
            c = 1.0 / sqrt(tt * tt + 1.0);
            s = tt * c;
          }
        }
        cs[i] = c;
        sn[i] = s;
        pp[i] = p;
        qq[i] = q < l ? q : -1;
      }
      __syncthreads();
      // columns: G <- G J, V <- V J
      for (int e = t; e < (n / 2) * l; e += nt) {
        const int i = e / l, k = e % l;
        const int p = pp[i], q = qq[i];
        if (q < 0) continue;
        const double c = cs[i], s = sn[i];
        const double gp = G[k * l + p], gq = G[k * l + q];
        G[k * l + p] = c * gp - s * gq;
        G[k * l + q] = s * gp + c * gq;
        const double vp = V[k * l + p], vq = V[k * l + q];
        V[k * l + p] = c * vp - s * vq;
        V[k * l + q] = s * vp + c * vq;
      }
      __syncthreads();
      // rows: G <- J^T G
      for (int e = t; e < (n / 2) * l; e += nt) {
        const int i = e / l, k = e % l;
        const int p = pp[i], q = qq[i];
        if (q < 0) continue;
        const double c = cs[i], s = sn[i];
        const double gp = G[p * l + k], gq = G[q * l + k];
        G[p * l + k] = c * gp - s * gq;
        G[q * l + k] = s * gp + c * gq;
      }
      __syncthreads();
    }
  }
  if (t == 0) {
    for (int i = 0; i < l; ++i) order[i] = i;
    for (int i = 0; i < l; ++i) {   // selection sort, descending, stable
      int best = i;
      for (int j = i + 1; j < l; ++j)
        if (G[order[j] * l + order[j]] > G[order[best] * l + order[best]]) best = j;
      const int x = order[best];
      for (int j = best; j > i; --j) order[j] = order[j - 1];
      order[i] = x;
    }
  }
  __syncthreads();
  for (int e = t; e < l * l; e += nt) {
    const int k = e / l, j = e % l;
    const double v = V[k * l + order[j]];
    if (!isfinite(v)) set_flag(status, TTQ_FLAG_NONFINITE);
    U[e] = static_cast<float>(v);
  }
  const double lam0 = G[order[0] * l + order[0]];
  const double smax = lam0 > 0.0 ? sqrt(lam0) : 0.0;
  for (int j = t; j < l; j += nt) {
    const double lam = G[order[j] * l + order[j]];
    const double s = lam > 0.0 ? sqrt(lam) : 0.0;
    sigma[j] = static_cast<float>(s);
    inv_sigma[j] = (s > 1e-6 * smax && s > 0.0) ? static_cast<float>(1.0 / s) : 0.f;
  }
}

template <typename TA, typename TB>
cudaError_t run_product(GemmView g, const TA* A, const TB* B, int num_sms, cudaStream_t stream) {
  if (g.M == 0 || g.N == 0) return cudaSuccess;
  const unsigned gm = static_cast<unsigned>((g.M + kTM - 1) / kTM);
  const unsigned gn = static_cast<unsigned>((g.N + kTN - 1) / kTN);
  const dim3 grid(gm, gn, static_cast<unsigned>(g.splits));
  strided_gemm_kernel<TA, TB><<<grid, kGemmThreads, 0, stream>>>(g, A, B);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || g.splits == 1) return e;
  const int64_t mn = g.M * g.N;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((mn + 255) / 256, 4 * num_sms));
  finish_split_kernel<<<blocks, 256, 0, stream>>>(g);
  return cudaGetLastError();
}

// A view with the split chosen to fill about two waves when the output
// has few tiles and the reduction is long.
GemmView make_view(int64_t M, int64_t N, int64_t K, int64_t sam, int64_t sak, int64_t sbk, int64_t sbn,
                   float* partial, int64_t partial_cap, int num_sms) {
  GemmView g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.sam = sam;
  g.sak = sak;
  g.sbk = sbk;
  g.sbn = sbn;
  const int64_t tiles = ((M + kTM - 1) / kTM) * ((N + kTN - 1) / kTN);
  int64_t splits = 1;
  if (partial != nullptr && tiles < 2 * num_sms) {
    splits = (2 * num_sms + tiles - 1) / tiles;
    splits = std::min<int64_t>(splits, std::max<int64_t>(1, K / 256));
    splits = std::min<int64_t>(splits, 256);
    while (splits > 1 && splits * M * N > partial_cap) --splits;
  }
  g.splits = static_cast<int>(splits);
  g.kps = (K + splits - 1) / splits;
  g.kps = (g.kps + kTK - 1) / kTK * kTK;
  g.partial = partial;
  g.out_type = 0;
  return g;
}

}  // namespace

LowrankLayout lowrank_layout(int64_t dp, int64_t d, int64_t l) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  LowrankLayout L{};
  size_t off = 4096;   // status word and reserve
  const int64_t rows = std::max(dp, d);
  L.Y = off;
  off = up(off + 4 * static_cast<size_t>(rows) * l);
  L.Q = off;
  off = up(off + 4 * static_cast<size_t>(rows) * l);
  L.Bt = off;
  off = up(off + 4 * static_cast<size_t>(d) * l);
  L.partial_floats = std::max<int64_t>(static_cast<int64_t>(l) * l * 256, 1);
  L.partial = off;
  off = up(off + 4 * static_cast<size_t>(L.partial_floats));
  L.G = off;
  off = up(off + 8 * static_cast<size_t>(l) * l);
  L.Rinv = off;
  off = up(off + 4 * static_cast<size_t>(l) * l);
  L.U = off;
  off = up(off + 4 * static_cast<size_t>(l) * l);
  L.sigma = off;
  off = up(off + 4 * static_cast<size_t>(l));
  L.inv_sigma = off;
  off = up(off + 4 * static_cast<size_t>(l));
  L.total = off;
  return L;
}

size_t lowrank_small_smem(int l, bool eig) {
  const size_t n = static_cast<size_t>((l + 1) & ~1);
  return eig ? 16 * static_cast<size_t>(l) * l + 8 * n + 4 * n + 4 * static_cast<size_t>(l)
             : 16 * static_cast<size_t>(l) * l;
}

cudaError_t launch_lowrank_init(const void* W, bool w_bf16, int64_t dp, int64_t d, int64_t r, int64_t l,
                                int power_iters, const float* Omega, void* Bout, void* Aout, void* Wres,
                                void* ws, int num_sms, cudaStream_t stream) {
  const LowrankLayout L = lowrank_layout(dp, d, l);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  float* Y = reinterpret_cast<float*>(base + L.Y);
  float* Q = reinterpret_cast<float*>(base + L.Q);
  float* Bt = reinterpret_cast<float*>(base + L.Bt);
  float* part = reinterpret_cast<float*>(base + L.partial);
  double* G = reinterpret_cast<double*>(base + L.G);
  float* Rinv = reinterpret_cast<float*>(base + L.Rinv);
  float* Us = reinterpret_cast<float*>(base + L.U);
  float* sig = reinterpret_cast<float*>(base + L.sigma);
  float* isig = reinterpret_cast<float*>(base + L.inv_sigma);
  const size_t chol_smem = lowrank_small_smem(static_cast<int>(l), false);
  const size_t eig_smem = lowrank_small_smem(static_cast<int>(l), true);
  cudaError_t e = cudaFuncSetAttribute(chol_rinv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(chol_smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(eig_smem));
  if (e != cudaSuccess) return e;

  // W as the left operand (W X: sam = d, sak = 1) or transposed (W^T X:
  // sam = 1, sak = d), through either element type
  auto with_w = [&](GemmView g, const float* Bop) -> cudaError_t {
    return w_bf16 ? run_product(g, static_cast<const __nv_bfloat16*>(W), Bop, num_sms, stream)
                  : run_product(g, static_cast<const float*>(W), Bop, num_sms, stream);
  };
  // orth: the rows x l matrix in src, orthonormalised into dst (shifted
  // CholeskyQR3: src -> dst -> src -> dst; src is overwritten)
  auto orth = [&](float* src, float* dst, int64_t rows) -> cudaError_t {
    float* cur = src;
    float* nxt = dst;
    for (int pass = 0; pass < 3; ++pass) {
      GemmView gg = make_view(l, l, rows, 1, l, l, 1, part, L.partial_floats, num_sms);
      gg.out = G;
      gg.out_type = 2;
      gg.som = l;
      gg.son = 1;
      cudaError_t err = run_product(gg, cur, cur, num_sms, stream);
      if (err != cudaSuccess) return err;
      chol_rinv_kernel<<<1, 256, chol_smem, stream>>>(G, static_cast<int>(l), pass == 0 ? 1e-6 : 0.0,
                                                      Rinv, status);
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
      GemmView gq = make_view(rows, l, l, l, 1, l, 1, nullptr, 0, num_sms);
      gq.out = nxt;
      gq.som = l;
      gq.son = 1;
      if ((err = run_product(gq, cur, Rinv, num_sms, stream)) != cudaSuccess) return err;
      float* x = cur;
      cur = nxt;
      nxt = x;
    }
    return cudaSuccess;
  };
  // W X (dp x l) and W^T X (d x l) for an l-column X, into out
  auto w_times = [&](const float* X, float* out) -> cudaError_t {
    GemmView gw = make_view(dp, l, d, d, 1, l, 1, nullptr, 0, num_sms);
    gw.out = out;
    gw.som = l;
    gw.son = 1;
    return with_w(gw, X);
  };
  auto wt_times = [&](const float* X, float* out) -> cudaError_t {
    GemmView gw = make_view(d, l, dp, 1, d, l, 1, nullptr, 0, num_sms);
    gw.out = out;
    gw.som = l;
    gw.son = 1;
    return with_w(gw, X);
  };

  // Q = orth(W Omega): Y buffer -> Q buffer
  float* Qp = Q;       // holds the current orthonormal basis of W's range
  float* other = Y;
  if ((e = w_times(Omega, Y)) != cudaSuccess) return e;
  if ((e = orth(Y, Q, dp)) != cudaSuccess) return e;
  for (int it = 0; it < power_iters; ++it) {
    // Z = orth(W^T Q) (d x l, in `other`); then Q = orth(W Z)
    if ((e = wt_times(Qp, Bt)) != cudaSuccess) return e;
    if ((e = orth(Bt, other, d)) != cudaSuccess) return e;
    if ((e = w_times(other, Qp)) != cudaSuccess) return e;
    if ((e = orth(Qp, other, dp)) != cudaSuccess) return e;
    float* x = Qp;
    Qp = other;
    other = x;
  }
  // Bt = W^T Q (d x l), then its Gram matrix and eigendecomposition
  if ((e = wt_times(Qp, Bt)) != cudaSuccess) return e;
  GemmView g = make_view(l, l, d, 1, l, l, 1, part, L.partial_floats, num_sms);
  g.out = G;
  g.out_type = 2;
  g.som = l;
  g.son = 1;
  if ((e = run_product(g, Bt, Bt, num_sms, stream)) != cudaSuccess) return e;
  jacobi_eig_kernel<<<1, 512, eig_smem, stream>>>(G, static_cast<int>(l), Us, sig, isig, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int out_type = w_bf16 ? 1 : 0;
  // B = Q U~_r diag(sigma_r)  (d' x r)
  g = make_view(dp, r, l, l, 1, l, 1, nullptr, 0, num_sms);
  g.col_scale = sig;
  g.out = Bout;
  g.out_type = out_type;
  g.som = r;
  g.son = 1;
  if ((e = run_product(g, Qp, Us, num_sms, stream)) != cudaSuccess) return e;
  // A^T = Bt U~_r diag(1 / sigma_r) (d x r), stored transposed as A (r x d)
  g = make_view(d, r, l, l, 1, l, 1, nullptr, 0, num_sms);
  g.col_scale = isig;
  g.out = Aout;
  g.out_type = out_type;
  g.som = 1;
  g.son = d;
  if ((e = run_product(g, Bt, Us, num_sms, stream)) != cudaSuccess) return e;
  if (Wres == nullptr) return cudaSuccess;
  // W_res = W - B A with the stored B, A
  g = make_view(dp, d, r, r, 1, d, 1, nullptr, 0, num_sms);
  g.sub = W;
  g.sub_bf16 = w_bf16 ? 1 : 0;
  g.ssm = d;
  g.ssn = 1;
  g.out = Wres;
  g.out_type = out_type;
  g.som = d;
  g.son = 1;
  return w_bf16 ? run_product(g, static_cast<const __nv_bfloat16*>(Bout),
                              static_cast<const __nv_bfloat16*>(Aout), num_sms, stream)
                : run_product(g, static_cast<const float*>(Bout), static_cast<const float*>(Aout),
                              num_sms, stream);
}

}  // namespace ttq
