// Steps (2)-(3) of the TTQ layer on the 5th-generation tensor cores:
//   Y[t][j] = sum_i W_hat[j][i] X[t][i]  (+ sum_k B[j][k] AX[t][k])
// with W_hat[j][i] = s_jk (q_ji - z_jk) D_ii^(-1/2)
// (gist.science/zh/paper/2603.19296, section 2.1 for W_hat, 2.2 for the
// static low-rank pair, 2.3 for the projection).
//
// One CTA computes a 128 (rows of W) x BN (tokens) tile of Y^T in tensor
// memory with tcgen05.mma kind::f16 (binary16 x binary16 -> fp32 for the
// quantised weight; bf16 x bf16 for the low-rank tail), cta_group::1:
//   warp 0      TMA producer: X tiles (BN x 64, 128-byte swizzle) into the
//               B slot of each pipeline stage; in the plain mode (no codes)
//               and for the low-rank tail also the A slot.
//   warp 1      allocates tensor memory; one lane issues the MMAs and
//               commits each stage back to its "empty" barrier.
//   warps 2-9   dequantise packed codes straight into the A slot, written in
//               the same 128-byte-swizzled K-major layout the TMA produces,
//               then (after the last stage) read the accumulator out of
//               tensor memory and store Y.
// W_hat is formed in fp32 -- (q - z) * s is exact, one rounding for the
// D^(-1/2) factor -- and rounded once to binary16 (11 significant bits; a
// bf16 W_hat would carry 8x the rounding error on the few large
// outlier-channel terms).  X arrives as binary16, exact for bf16 inputs of
// magnitude <= 65504.  The low-rank term rides along as extra K blocks: A
// slot = B[j][k] (TMA), B slot = AX[t][k] (TMA), both bf16.
//
// Every barrier wait is bounded (1 s); a wait that gives up sets
// TTQ_FLAG_TIMEOUT, tells the other roles to stop, and the CTA still frees
// its tensor memory and returns.
#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;                        // bf16 elements per 128-byte row
constexpr int kATileBytes = kBM * kBK * 2;     // 16 KiB
constexpr int kThreads = 320;
constexpr int kProducerWarps = 8;
constexpr int kMaxStages = 6;
constexpr int kSmemLimit = 232448;             // 227 KiB opt-in per block

struct GemmDev {
  const uint32_t* codes;
  const __half* scales;
  const __half* zeros;
  const float* Dr;
  int group;
  int64_t K, M, T, K_tail;
  void* Y;
  int64_t ldy;
  int y_f32;
  int BN;
  int stages;
  uint32_t* status;
};

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Writes rows rb, rb+32, rb+64, rb+96 of the 128 x 64 A tile, channels
// [8c, 8c+8) of K block kb, as binary16 W_hat in the 128-byte-swizzled layout:
// row r, 16-byte chunk c lives at (r/8)*1024 + (r%8)*128 + ((c ^ r%8) * 16).
template <int BITS>
__device__ __forceinline__ void dequant_rows(uint32_t a_slot, const GemmDev& g, int64_t m0,
                                             int kb, int c, int rb) {
  constexpr int QMAX = (1 << BITS) - 1;
  const int64_t col = static_cast<int64_t>(kb) * kBK + c * 8;
  const bool col_ok = col < g.K;  // K % 8 == 0: the 8 channels are all in or all out
  float dr[8];
  if (col_ok && g.Dr != nullptr) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(g.Dr + col));
    const float4 b = __ldg(reinterpret_cast<const float4*>(g.Dr + col) + 1);
    dr[0] = a.x; dr[1] = a.y; dr[2] = a.z; dr[3] = a.w;
    dr[4] = b.x; dr[5] = b.y; dr[6] = b.z; dr[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) dr[e] = 1.0f;
  }
  const int64_t ng = g.K / g.group;
  const int64_t wpr = g.K * BITS / 32;
  const int64_t k = col / g.group;
  const int64_t bitoff = col * BITS;
  const int64_t widx = bitoff >> 5;
  const int sh = static_cast<int>(bitoff & 31);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = rb + 32 * u;
    const int64_t row = m0 + r;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (col_ok && row < g.M) {
      const uint32_t* crow = g.codes + row * wpr;
      uint32_t v = __ldg(crow + widx) >> sh;
      if (BITS == 3 && sh > 8) v |= __ldg(crow + widx + 1) << (32 - sh);
      const float s = __half2float(g.scales[row * ng + k]);
      const int z = static_cast<int>(__half2float(g.zeros[row * ng + k]));
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int q = static_cast<int>((v >> (BITS * e)) & QMAX);
        w[e] = __fmul_rn(static_cast<float>(q - z) * s, dr[e]);
      }
      out.x = pack_f16x2(w[0], w[1]);
      out.y = pack_f16x2(w[2], w[3]);
      out.z = pack_f16x2(w[4], w[5]);
      out.w = pack_f16x2(w[6], w[7]);
    }
    const uint32_t addr = a_slot + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
    st_shared_v4(addr, out);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    ttq_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                    const GemmDev g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int BN = g.BN;
  const int stages = g.stages;
  const int stage_bytes = kATileBytes + BN * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* accum = empty + kMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * BN;
  const int kb_main = static_cast<int>((g.K + kBK - 1) / kBK);
  const int kb_tail = static_cast<int>((g.K_tail + kBK - 1) / kBK);
  const int kb_total = kb_main + kb_tail;
  const uint32_t tmem_cols = BN <= 32 ? 32u : BN <= 64 ? 64u : BN <= 128 ? 128u : 256u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1 + kProducerWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmB0);
    if (BITS == 0) prefetch_tensormap(&tmA0);
    if (kb_tail > 0) {
      prefetch_tensormap(&tmA1);
      prefetch_tensormap(&tmB1);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int kb = 0; kb < kb_total; ++kb) {
        const int s = kb % stages;
        const uint32_t ph = static_cast<uint32_t>(kb / stages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
          break;
        }
        uint8_t* a_slot = smem + s * stage_bytes;
        uint8_t* b_slot = a_slot + kATileBytes;
        if (kb < kb_main) {
          const uint32_t bytes = BN * 128 + (BITS == 0 ? kATileBytes : 0);
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(&tmB0, &full[s], b_slot, kb * kBK, static_cast<int32_t>(n0));
          if (BITS == 0) tma_load_2d(&tmA0, &full[s], a_slot, kb * kBK, static_cast<int32_t>(m0));
        } else {
          const int kt = (kb - kb_main) * kBK;
          mbar_arrive_expect_tx(&full[s], BN * 128 + kATileBytes);
          tma_load_2d(&tmB1, &full[s], b_slot, kt, static_cast<int32_t>(n0));
          tma_load_2d(&tmA1, &full[s], a_slot, kt, static_cast<int32_t>(m0));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // main K blocks: binary16 W_hat x binary16 X (bf16 x bf16 in the plain
      // mode); low-rank tail: bf16 B x bf16 A X
      const uint32_t idesc_main =
          idesc_f16kind(BITS == 0 ? kFmtBF16 : kFmtF16, kBM, static_cast<uint32_t>(BN));
      const uint32_t idesc_tail = idesc_f16kind(kFmtBF16, kBM, static_cast<uint32_t>(BN));
      for (int kb = 0; kb < kb_total; ++kb) {
        const int s = kb % stages;
        const uint32_t ph = static_cast<uint32_t>(kb / stages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_addr(smem + s * stage_bytes);
        const uint64_t adesc = smem_desc_sw128(a_addr);
        const uint64_t bdesc = smem_desc_sw128(a_addr + kATileBytes);
        const uint32_t idesc = kb < kb_main ? idesc_main : idesc_tail;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          mma_f16kind_ss(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
    __syncwarp();
  } else {
    // ------------------------------------- dequant producers + epilogue
    const int pt = threadIdx.x - 64;  // 0..255
    const int c = pt & 7;
    const int rb = pt >> 3;
    for (int kb = 0; kb < kb_total; ++kb) {
      const int s = kb % stages;
      const uint32_t ph = static_cast<uint32_t>(kb / stages) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
        }
        break;
      }
      if (BITS != 0 && kb < kb_main) {
        dequant_rows<(BITS == 0 ? 4 : BITS)>(smem_addr(smem + s * stage_bytes), g, m0, kb, c, rb);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
    }

    int ok = 1;
    if (lane == 0) ok = mbar_wait(accum, 0, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_flag(g.status, TTQ_FLAG_TIMEOUT);
    }
    tc_fence_after_sync();
    const int q = warp & 3;             // tensor-memory lane quadrant of this warp
    const int half = (warp - 2) >> 2;   // two warps per quadrant split the columns
    const int64_t j = m0 + q * 32 + lane;
    const int nchunks = BN / 16;
    const bool store = ok && (*abort_flag == 0) && j < g.M;
    for (int ch = half; ch < nchunks; ch += 2) {
      uint32_t r[16];
      tmem_load_16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ch * 16, r);
      tmem_load_wait();
      if (store) {
        const int64_t t0 = n0 + ch * 16;
        if (g.y_f32) {
          float* Y = static_cast<float*>(g.Y);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (t0 + i < g.T) Y[(t0 + i) * g.ldy + j] = __uint_as_float(r[i]);
        } else {
          __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(g.Y);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (t0 + i < g.T) Y[(t0 + i) * g.ldy + j] = __float2bfloat16_rn(__uint_as_float(r[i]));
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

template <int BITS>
cudaError_t launch_bits(const GemmArgs& a, const GemmMaps& maps, int BN, cudaStream_t stream) {
  const int stage_bytes = kATileBytes + BN * 128;
  int stages = (kSmemLimit - 2048) / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  const int smem = stages * stage_bytes + 2048;
  cudaError_t err = cudaFuncSetAttribute(ttq_gemm_kernel<BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  GemmDev g;
  g.codes = a.codes;
  g.scales = reinterpret_cast<const __half*>(a.scales);
  g.zeros = reinterpret_cast<const __half*>(a.zeros);
  g.Dr = a.Dr;
  g.group = a.group;
  g.K = a.K;
  g.M = a.M;
  g.T = a.T;
  g.K_tail = a.K_tail;
  g.Y = a.Y;
  g.ldy = a.ldy;
  g.y_f32 = a.y_f32 ? 1 : 0;
  g.BN = BN;
  g.stages = stages;
  g.status = a.status;
  const dim3 grid(static_cast<unsigned>((a.M + kBM - 1) / kBM),
                  static_cast<unsigned>((a.T + BN - 1) / BN));
  ttq_gemm_kernel<BITS><<<grid, kThreads, smem, stream>>>(maps.a0, maps.b0, maps.a1, maps.b1, g);
  return cudaGetLastError();
}

}  // namespace

int gemm_block_n(int64_t T) {
  if (T >= 256) return 256;
  int64_t bn = (T + 15) / 16 * 16;
  if (bn < 16) bn = 16;
  return static_cast<int>(bn);
}

cudaError_t launch_dequant_gemm(const GemmArgs& args, const GemmMaps& maps, int block_n,
                                cudaStream_t stream) {
  if (args.M == 0 || args.T == 0) return cudaSuccess;
  if (block_n % 16 != 0 || block_n < 16 || block_n > 256) return cudaErrorInvalidValue;
  switch (args.bits) {
    case 0:
      return launch_bits<0>(args, maps, block_n, stream);
    case 2:
      return launch_bits<2>(args, maps, block_n, stream);
    case 3:
      return launch_bits<3>(args, maps, block_n, stream);
    case 4:
      return launch_bits<4>(args, maps, block_n, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ttq
