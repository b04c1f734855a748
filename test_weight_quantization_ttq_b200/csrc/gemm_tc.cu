// Steps (2)-(3) of the TTQ layer on the 5th-generation tensor cores:
//   Y[t][j] = sum_i W_hat[j][i] X[t][i]  (+ sum_k B[j][k] AX[t][k])
// with W_hat[j][i] = s_jk (q_ji - z_jk) D_ii^(-1/2)
// (gist.science/zh/paper/2603.19296, section 2.1 for W_hat, 2.2 for the
// static low-rank pair, 2.3 for the projection).
//
// One CTA computes a BM (rows of W: 128 or 256) x BN (tokens) tile of Y^T in
// tensor memory with tcgen05.mma kind::f16 (binary16 x binary16 -> fp32 for
// the quantised weight; bf16 x bf16 for the low-rank tail), cta_group::1; a
// 256-row tile is two 128-row MMAs that share each X tile, which halves the
// X traffic per FLOP:
//   warp 0      TMA producer: X tiles (BN x 64, 128-byte swizzle) into the
//               B slot of each pipeline stage; in the plain mode (no codes)
//               and for the low-rank tail also the A slot.
//   warp 1      allocates tensor memory; one lane issues the MMAs and
//               commits each stage back to its "empty" barrier.
//   warps 2..   two threads per tile row (8 or 16 warps) dequantise packed
//               codes straight into the A slot, written in the same
//               128-byte-swizzled K-major layout the TMA produces, then
//               (after the last stage) read the accumulator out of tensor
//               memory and store Y.
// The factor D^(-1/2) of W_hat is carried by the B operand, which arrives
// as binary16 X D^(-1/2); the A operand is s (q - z), built in binary16 with
// integer-free bit tricks ((1024 + q) from the code bits, minus (1024 + z),
// times s: exact until the one rounding of the product).  Binary16 keeps 11
// significant bits, where bf16 operands would carry 8x the rounding error on
// the few large outlier-channel terms.  The low-rank term rides along as
// extra K blocks: A slot = B[j][k] (TMA), B slot = AX[t][k] (TMA), both bf16.
//
// Every barrier wait is bounded (1 s); a wait that gives up sets
// TTQ_FLAG_TIMEOUT, tells the other roles to stop, and the CTA still frees
// its tensor memory and returns.
#include <algorithm>

#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int kBK = 64;                        // 16-bit elements per 128-byte row
constexpr int kSubTileBytes = 128 * kBK * 2;   // one 128-row operand tile: 16 KiB
// Threads of a CTA: warp 0 (TMA), warp 1 (MMA), then two producer /
// epilogue threads per row of the tile.
template <int BM>
constexpr int cta_threads() { return 64 + 2 * BM; }
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;             // 227 KiB opt-in per block

struct GemmDev {
  const uint32_t* codes;
  const uint16_t* scales;
  const uint16_t* zeros;
  int group_shift;      // log2(group): groups are powers of two
  int64_t ngroups;      // K / group
  int sz_shift;         // scales/zeros are loaded 2^sz_shift groups at a time (<= 8)
  int64_t K, M, T, K_tail;
  void* Y;
  int64_t ldy;
  int y_f32;
  int y_tma;            // bf16 Y written by TMA stores of 32 x 16 slabs (tmY)
  int a_f16;            // plain mode: binary16 A operand (else bf16)
  int BN;
  int stages;
  int kb_per_split;     // split-K: K blocks per split (0: no split)
  int64_t split_stride; // split-K: elements between the splits' partial outputs
  uint32_t* status;
};

__device__ __forceinline__ __half2 u2h(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return h;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) {
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// The operands one producer thread needs for one K block: the packed codes
// of its 32 channels of one row, and that row's scale and zero point.
struct CodeChunk {
  uint32_t w[4];
  uint16_t s, z;
};

// Loads the chunk of row `row`, channels [col0, col0 + 32) (zeros outside W).
template <int BITS>
__device__ __forceinline__ void load_chunk(const GemmDev& g, int64_t row, int64_t col0,
                                           CodeChunk& ck) {
  ck.w[0] = ck.w[1] = ck.w[2] = ck.w[3] = 0u;
  ck.s = 0;
  ck.z = 0;
  if (row >= g.M || col0 >= g.K) return;
  const int64_t wpr = g.K * BITS / 32;
  const uint32_t* crow = g.codes + row * wpr + (col0 >> 5) * BITS;
  if (BITS == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(crow));
    ck.w[0] = v.x; ck.w[1] = v.y; ck.w[2] = v.z; ck.w[3] = v.w;
  } else if (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(crow));
    ck.w[0] = v.x; ck.w[1] = v.y;
  } else {
    ck.w[0] = __ldg(crow);
    ck.w[1] = __ldg(crow + 1);
    ck.w[2] = __ldg(crow + 2);
  }
  const int64_t gi = row * g.ngroups + (col0 >> g.group_shift);
  ck.s = __ldg(g.scales + gi);
  ck.z = __ldg(g.zeros + gi);
}

// Reads the packed codes of one 32-channel chunk from the K block's code
// tile in shared memory (rows of cw words, first needed word at `off`).
template <int BITS>
__device__ __forceinline__ void read_codes_smem(uint32_t row_addr, int hf, CodeChunk& ck) {
  if (BITS == 4) {
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(ck.w[0]), "=r"(ck.w[1]), "=r"(ck.w[2]), "=r"(ck.w[3])
                 : "r"(row_addr + 16 * hf));
  } else if (BITS == 2) {
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                 : "=r"(ck.w[0]), "=r"(ck.w[1])
                 : "r"(row_addr + 8 * hf));
  } else {
#pragma unroll
    for (int i = 0; i < 3; ++i)
      asm volatile("ld.shared.b32 %0, [%1];" : "=r"(ck.w[i]) : "r"(row_addr + 12 * hf + 4 * i));
  }
}

// Per-thread cache of one row's scales and zero points, 2^sz_shift groups
// per load (the largest of 8, 4, 2, 1 that divides K/group, so every load is
// aligned): `cur` holds group block gb, `nxt` the block after it, loaded
// one block ahead so its latency is hidden.
struct SZCache {
  int64_t gb;
  uint4 s_cur, z_cur, s_nxt, z_nxt;
};

__device__ __forceinline__ void sz_load(const GemmDev& g, int64_t row, int64_t gb, uint4& sv,
                                        uint4& zv) {
  sv = make_uint4(0u, 0u, 0u, 0u);
  zv = sv;
  const int64_t k0 = gb << g.sz_shift;
  if (row >= g.M || k0 >= g.ngroups) return;
  const int64_t i = row * g.ngroups + k0;
  switch (g.sz_shift) {
    case 3:
      sv = __ldg(reinterpret_cast<const uint4*>(g.scales + i));
      zv = __ldg(reinterpret_cast<const uint4*>(g.zeros + i));
      break;
    case 2: {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(g.scales + i));
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(g.zeros + i));
      sv.x = a.x; sv.y = a.y; zv.x = b.x; zv.y = b.y;
      break;
    }
    case 1:
      sv.x = __ldg(reinterpret_cast<const uint32_t*>(g.scales + i));
      zv.x = __ldg(reinterpret_cast<const uint32_t*>(g.zeros + i));
      break;
    default:
      sv.x = __ldg(g.scales + i);
      zv.x = __ldg(g.zeros + i);
  }
}

__device__ __forceinline__ uint16_t u16_at(const uint4& v, int idx) {
  const int w = idx >> 1;
  const uint32_t word = w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
  return static_cast<uint16_t>(word >> (16 * (idx & 1)));
}

// Scale and zero of group k (k lies in block gb or gb + 1 of the cache).
__device__ __forceinline__ void sz_get(const GemmDev& g, const SZCache& c, int64_t k, uint16_t& sc,
                                       uint16_t& ze) {
  const int64_t blk = k >> g.sz_shift;
  const int idx = static_cast<int>(k - (blk << g.sz_shift));
  const bool in_cur = blk == c.gb;
  sc = u16_at(in_cur ? c.s_cur : c.s_nxt, idx);
  ze = u16_at(in_cur ? c.z_cur : c.z_nxt, idx);
}

// (1024 + q) in both halves of a half2 from two codes placed at bits [0, b)
// and [16, 16 + b) of `bits`.  0x6400 is binary16 1024.0, whose unit in the
// last place is 1, so OR-ing a code into the fraction adds it exactly.
__device__ __forceinline__ uint32_t magic_pair(uint32_t bits) { return bits | 0x64006400u; }

// Writes the 32 channels of one row, 32-channel half `hf` of the K block, as
// binary16 s (q - z) into the 128-byte-swizzled A tile: in a 128-row
// sub-tile, row r's 16-byte chunk c lives at (r/8)*1024 + (r%8)*128 +
// ((c ^ r%8) * 16); row_base is the row's address and rsw = r % 8.  (q - z)
// is exact in binary16, the product is rounded once; D^(-1/2) is carried by
// X.
template <int BITS>
__device__ __forceinline__ void dequant_chunk(uint32_t row_base, int rsw, int hf,
                                              const CodeChunk& ck) {
  const __half2 c2 = __half2half2(__hadd(__ushort_as_half(ck.z), __ushort_as_half(0x6400)));
  const __half2 s2 = __half2half2(__ushort_as_half(ck.s));
  auto put = [&](int chunk, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    st_shared_v4(row_base + (((4 * hf + chunk) ^ rsw) << 4), a, b, c, d);
  };
  auto val = [&](uint32_t pairbits) { return h2u(__hmul2(__hsub2(u2h(magic_pair(pairbits)), c2), s2)); };
  if (BITS == 4 || BITS == 3) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // y holds codes 0-3 of this 8-code group in bits 0-15 and codes 4-7 in
      // bits 16-31, each at 4-bit (INT4) or 3-bit (INT3) spacing
      uint32_t y;
      if (BITS == 4) {
        y = ck.w[i];
      } else {
        // the 24 bits of codes 8i..8i+7 start at bit 24i of the 96-bit row piece
        const int wi = (24 * i) >> 5;
        const uint32_t v =
            __funnelshift_r(ck.w[wi], ck.w[wi + 1 < 3 ? wi + 1 : 2], (24 * i) & 31) & 0xFFFFFFu;
        y = (v & 0xFFFu) | ((v << 4) & 0x0FFF0000u);
      }
      constexpr uint32_t M = BITS == 4 ? 0x000F000Fu : 0x00070007u;
      const uint32_t h0 = val(y & M);                       // (q0, q4)
      const uint32_t h1 = val((y >> BITS) & M);             // (q1, q5)
      const uint32_t h2 = val((y >> (2 * BITS)) & M);       // (q2, q6)
      const uint32_t h3 = val((y >> (3 * BITS)) & M);       // (q3, q7)
      put(i, __byte_perm(h0, h1, 0x5410), __byte_perm(h2, h3, 0x5410), __byte_perm(h0, h1, 0x7632),
          __byte_perm(h2, h3, 0x7632));
    }
  } else {  // BITS == 2: two words of 16 codes, each filling two chunks
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w = ck.w[k];
      uint32_t h[8];  // h[e] = (q_e, q_{e+8})
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = val((w >> (2 * e)) & 0x00030003u);
      put(2 * k, __byte_perm(h[0], h[1], 0x5410), __byte_perm(h[2], h[3], 0x5410),
          __byte_perm(h[4], h[5], 0x5410), __byte_perm(h[6], h[7], 0x5410));
      put(2 * k + 1, __byte_perm(h[0], h[1], 0x7632), __byte_perm(h[2], h[3], 0x7632),
          __byte_perm(h[4], h[5], 0x7632), __byte_perm(h[6], h[7], 0x7632));
    }
  }
}

// Words of packed codes per row that the TMA brings in for one K block
// (INT3 reads a 16-byte-aligned window of 8 words that holds the 6 needed).
template <int BITS>
constexpr int code_tile_words() { return BITS == 2 ? 4 : 8; }

template <int BITS, int BM, bool TC>
__global__ void __launch_bounds__(cta_threads<BM>(), 1)
    ttq_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
                    const GemmDev g) {
  constexpr int kSub = BM / 128;                 // 128-row MMAs per K step
  constexpr int kProducerWarps = BM / 16;        // 2 threads per tile row
  constexpr int kATile = BM * kBK * 2;
  constexpr int kCW = code_tile_words<BITS == 0 ? 4 : BITS>();
  constexpr int kCTile = TC ? BM * kCW * 4 : 0;  // code tile of one K block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int BN = g.BN;
  const int stages = g.stages;
  const int stage_bytes = kATile + BN * 128 + kCTile;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* cfull = empty + kMaxStages;
  uint64_t* accum = cfull + kMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * BN;
  const int kb_main = static_cast<int>((g.K + kBK - 1) / kBK);
  const int kb_tail = static_cast<int>((g.K_tail + kBK - 1) / kBK);
  // this CTA's K blocks [kb_lo, kb_total): all of them, or one split of the
  // main blocks (split-K runs only in the plain mode); the last split takes
  // the rest of the main blocks and the low-rank tail
  const bool k_split = g.kb_per_split > 0;
  const int kb_lo = k_split ? static_cast<int>(blockIdx.z) * g.kb_per_split : 0;
  const int kb_total = !k_split || blockIdx.z + 1 == gridDim.z
                           ? kb_main + kb_tail
                           : min(kb_main, kb_lo + g.kb_per_split);
  // accumulator h of a 256-row tile starts at column 256 * h
  const uint32_t tmem_cols =
      kSub == 2 ? 512u : (BN <= 32 ? 32u : BN <= 64 ? 64u : BN <= 128 ? 128u : 256u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      // the producer warps take part only when they build the A operand
      mbar_init(&full[s], 1 + (BITS != 0 ? kProducerWarps : 0));
      mbar_init(&empty[s], 1);
      mbar_init(&cfull[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (g.y_tma) prefetch_tensormap(&tmY);
    prefetch_tensormap(&tmB0);
    if (BITS == 0) prefetch_tensormap(&tmA0);
    if (TC) prefetch_tensormap(&tmC);
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
  // everything above overlaps the previous kernel; its outputs (codes, X)
  // are read only after this
  allow_dependents_launch();
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int kb = kb_lo; kb < kb_total; ++kb, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
          break;
        }
        uint8_t* a_slot = smem + s * stage_bytes;
        uint8_t* b_slot = a_slot + kATile;
        if (kb < kb_main) {
          if (TC) {
            // code tile first: the producers wait for it, the MMA does not
            const int32_t xw = BITS == 3 ? ((6 * kb) & ~3) : kb * kCW;
            mbar_arrive_expect_tx(&cfull[s], kCTile);
            tma_load_2d(&tmC, &cfull[s], b_slot + BN * 128, xw, static_cast<int32_t>(m0));
          }
          const uint32_t bytes = BN * 128 + (BITS == 0 ? kATile : 0);
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(&tmB0, &full[s], b_slot, kb * kBK, static_cast<int32_t>(n0));
          if (BITS == 0) tma_load_2d(&tmA0, &full[s], a_slot, kb * kBK, static_cast<int32_t>(m0));
        } else {
          const int kt = (kb - kb_main) * kBK;
          mbar_arrive_expect_tx(&full[s], BN * 128 + kATile);
          tma_load_2d(&tmB1, &full[s], b_slot, kt, static_cast<int32_t>(n0));
          tma_load_2d(&tmA1, &full[s], a_slot, kt, static_cast<int32_t>(m0));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // main K blocks: binary16 W_hat x binary16 X D^(-1/2) (bf16 x bf16 in
      // the plain mode); low-rank tail: bf16 B x bf16 A X
      const uint32_t idesc_main = idesc_f16kind(
          (BITS != 0 || g.a_f16) ? kFmtF16 : kFmtBF16, 128, static_cast<uint32_t>(BN));
      const uint32_t idesc_tail = idesc_f16kind(kFmtBF16, 128, static_cast<uint32_t>(BN));
      int s = 0;
      uint32_t ph = 0;
      for (int kb = kb_lo; kb < kb_total; ++kb, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_addr(smem + s * stage_bytes);
        const uint64_t bdesc = smem_desc_sw128(a_addr + kATile);
        const uint32_t idesc = kb < kb_main ? idesc_main : idesc_tail;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
#pragma unroll
          for (int h = 0; h < kSub; ++h) {
            const uint64_t adesc = smem_desc_sw128(a_addr + h * kSubTileBytes);
            mma_f16kind_ss(tmem_base + 256u * h, adesc + 2u * k, bdesc + 2u * k, idesc,
                           (kb != kb_lo || k != 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
      }
      mma_commit(accum);
    }
    __syncwarp();
  } else {
    // ------------------------------------- dequant producers + epilogue
    // Thread pt owns row pt % BM and the 32-channel half pt / BM of each K
    // block.  A warp thus writes 32 consecutive rows of one 16-byte chunk
    // column: conflict-free.
    const int pt = threadIdx.x - 64;  // 0 .. 2*BM-1
    const int r = pt % BM;
    constexpr int kChunks = 1;
    const int hf0 = pt / BM;
    const int rl = r & 127;
    const int rsw = r & 7;
    const uint32_t row_off = (r >> 7) * kSubTileBytes + (rl >> 3) * 1024 + (rl & 7) * 128;
    constexpr int LB = BITS == 0 ? 4 : BITS;
    int s = 0;
    uint32_t ph = 0;
    bool alive = true;
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          set_flag(g.status, TTQ_FLAG_TIMEOUT);
        }
        alive = false;
      }
      return ok != 0;
    };
    auto next_stage = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      s = (s + 1 == stages) ? 0 : s + 1;
      ph ^= (s == 0);
    };
    if (BITS == 0) {
      // plain mode: the A operand comes by TMA; nothing to build
    } else if (TC) {
      // Codes arrive by TMA with the stage (cfull); scales and zeros come
      // from the per-thread cache, two blocks of groups in registers.
      SZCache cache;
      cache.gb = 0;
      if (BITS != 0) {
        sz_load(g, m0 + r, 0, cache.s_cur, cache.z_cur);
        sz_load(g, m0 + r, 1, cache.s_nxt, cache.z_nxt);
      }
      for (int kb = 0; kb < kb_total; ++kb) {
        if (!wait_bar(&empty[s], ph ^ 1u)) break;
        if (BITS != 0 && kb < kb_main) {
          const int64_t col_first = static_cast<int64_t>(kb) * kBK + 32 * hf0;
          while (((col_first >> g.group_shift) >> g.sz_shift) > cache.gb) {
            // moved into the next block of groups: shift the cache by one
            cache.gb += 1;
            cache.s_cur = cache.s_nxt;
            cache.z_cur = cache.z_nxt;
            sz_load(g, m0 + r, cache.gb + 1, cache.s_nxt, cache.z_nxt);
          }
          if (!wait_bar(&cfull[s], ph)) break;
          const uint8_t* stage_base = smem + s * stage_bytes;
          const uint32_t crow = smem_addr(stage_base + kATile + BN * 128) + r * kCW * 4 +
                                (BITS == 3 ? 4 * ((6 * kb) & 3) : 0);
          const uint32_t row_base = smem_addr(stage_base) + row_off;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            CodeChunk ck;
            ck.w[3] = 0u;
            read_codes_smem<LB>(crow, hf0 + c, ck);
            sz_get(g, cache, (col_first + 32 * c) >> g.group_shift, ck.s, ck.z);
            dequant_chunk<LB>(row_base, rsw, hf0 + c, ck);
          }
          fence_proxy_async_smem();
        }
        next_stage();
      }
    } else {
      // Codes, scales and zeros loaded by each thread from global memory,
      // three K blocks ahead; the ring is walked by a loop unrolled four
      // times, so no register copy forces an early wait on a load in flight.
      CodeChunk c0[kChunks], c1[kChunks], c2[kChunks], c3[kChunks];
      auto load_kb = [&](int kbl, CodeChunk(&dst)[kChunks]) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          load_chunk<LB>(g, m0 + r, static_cast<int64_t>(kbl) * kBK + 32 * (hf0 + c), dst[c]);
      };
      if (BITS != 0) {
        if (0 < kb_main) load_kb(0, c0);
        if (1 < kb_main) load_kb(1, c1);
        if (2 < kb_main) load_kb(2, c2);
      }
      // one K block: prefetch block kb + 3 into `pre`, dequantise `use`
      auto step = [&](int kb, CodeChunk(&use)[kChunks], CodeChunk(&pre)[kChunks]) {
        if (BITS != 0 && kb + 3 < kb_main) load_kb(kb + 3, pre);
        if (!wait_bar(&empty[s], ph ^ 1u)) return;
        if (BITS != 0 && kb < kb_main) {
          const uint32_t row_base = smem_addr(smem + s * stage_bytes) + row_off;
#pragma unroll
          for (int c = 0; c < kChunks; ++c) dequant_chunk<LB>(row_base, rsw, hf0 + c, use[c]);
          fence_proxy_async_smem();
        }
        next_stage();
      };
      for (int kb = 0; kb < kb_total && alive; kb += 4) {
        step(kb, c0, c3);
        if (kb + 1 < kb_total && alive) step(kb + 1, c1, c0);
        if (kb + 2 < kb_total && alive) step(kb + 2, c2, c1);
        if (kb + 3 < kb_total && alive) step(kb + 3, c3, c2);
      }
    }

    int ok = 1;
    if (lane == 0) {
      ok = mbar_wait(accum, 0, abort_flag) ? 1 : 0;
      if (!ok) {
        *abort_flag = 1;
        set_flag(g.status, TTQ_FLAG_TIMEOUT);
        // the MMA issuer commits `accum` after its loop even when it stops
        // early: wait for that (with a fresh limit, not cut short by the
        // abort) so that no MMA still writes the tensor memory freed below
        int never = 0;
        mbar_wait(accum, 0, &never);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    tc_fence_after_sync();
    // warp w may read tensor-memory lanes 32 (w % 4) .. +31.  BM = 128: the
    // two warps of a lane quadrant split the columns; BM = 256: warps 2-5
    // read accumulator 0 (rows 0-127), warps 6-9 accumulator 1.
    const int q = warp & 3;
    // lane quadrant q = warp % 4 holds BM/64 warps: one per accumulator and
    // per half of the token chunks
    const int wg = (warp - 2) >> 2;
    const int acc = wg % kSub;
    const int ch0 = wg / kSub;
    const int chs = 2;
    const int jl = acc * 128 + q * 32 + lane;  // row of W within the tile
    const int64_t j = m0 + jl;
    const int nchunks = BN / 16;
    const bool good = ok && (*abort_flag == 0);
    if (g.y_tma) {
      // bf16 Y: each warp converts its 32 rows x 16 tokens of a chunk into a
      // 1 KiB slab [t][j] of the (now idle) pipeline memory and one lane
      // sends it out with a TMA store, while the next chunk's tensor-memory
      // load is in flight.
      const int iters = (nchunks + chs - 1) / chs;
      const uint32_t slabs = smem_addr(smem) + static_cast<uint32_t>((warp - 2) * iters) * 1024u;
      const int32_t jx = static_cast<int32_t>(m0 + acc * 128 + q * 32);
      const uint32_t tcol = tmem_base + 256u * acc + (static_cast<uint32_t>(q * 32) << 16);
      uint32_t ra[16], rb[16];
      if (ch0 < nchunks) {
        tmem_load_16(tcol + ch0 * 16, ra);
        tmem_load_wait(ra);
      }
      int it = 0;
      for (int ch = ch0; ch < nchunks; ch += chs, ++it) {
        const bool more = ch + chs < nchunks;
        if (more) tmem_load_16(tcol + (ch + chs) * 16, rb);
        const uint32_t slab = slabs + static_cast<uint32_t>(it) * 1024u;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(ra[i]));
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(slab + (i * 32 + lane) * 2),
                       "h"(*reinterpret_cast<const uint16_t*>(&v))
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && good) {
          tma_store_2d(&tmY, slab, jx, static_cast<int32_t>(n0 + ch * 16));
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        if (more) {
          tmem_load_wait(rb);
#pragma unroll
          for (int i = 0; i < 16; ++i) ra[i] = rb[i];
        }
      }
      if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    } else {
      const bool store = good && j < g.M;
      const int64_t yoff = g.kb_per_split > 0 ? static_cast<int64_t>(blockIdx.z) * g.split_stride : 0;
      for (int ch = ch0; ch < nchunks; ch += chs) {
        uint32_t rr[16];
        tmem_load_16(tmem_base + 256u * acc + (static_cast<uint32_t>(q * 32) << 16) + ch * 16, rr);
        tmem_load_wait(rr);
        if (store) {
          const int64_t t0 = n0 + ch * 16;
          if (g.y_f32) {
            float* Y = static_cast<float*>(g.Y) + yoff;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (t0 + i < g.T) Y[(t0 + i) * g.ldy + j] = __uint_as_float(rr[i]);
          } else {
            __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(g.Y);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (t0 + i < g.T) Y[(t0 + i) * g.ldy + j] = __float2bfloat16_rn(__uint_as_float(rr[i]));
          }
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

template <int BITS, int BM, bool TC>
cudaError_t launch_tile(const GemmArgs& a, const GemmMaps& maps, int BN, cudaStream_t stream,
                        bool pdl) {
  const int stage_bytes =
      BM * kBK * 2 + BN * 128 + (TC ? BM * code_tile_words<BITS == 0 ? 4 : BITS>() * 4 : 0);
  int stages = (kSmemLimit - 2048) / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  const int smem = stages * stage_bytes + 2048;
  cudaError_t err = cudaFuncSetAttribute(ttq_gemm_kernel<BITS, BM, TC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  GemmDev g;
  g.codes = a.codes;
  g.scales = a.scales;
  g.zeros = a.zeros;
  g.group_shift = 0;
  while (a.group > 0 && (1 << (g.group_shift + 1)) <= a.group) ++g.group_shift;
  g.ngroups = a.group > 0 ? a.K / a.group : 0;
  g.sz_shift = 0;
  while (g.sz_shift < 3 && g.ngroups % (int64_t{2} << g.sz_shift) == 0) ++g.sz_shift;
  g.K = a.K;
  g.M = a.M;
  g.T = a.T;
  g.K_tail = a.K_tail;
  g.Y = a.Y;
  g.ldy = a.ldy;
  g.y_f32 = a.y_f32 ? 1 : 0;
  g.a_f16 = a.a_f16 ? 1 : 0;
  // the Y slabs (1 KiB per producer warp and chunk pair) must fit in the
  // pipeline memory
  const int slab_bytes = (2 * BM / 32) * ((BN / 16 + 1) / 2) * 1024;
  g.y_tma = (a.y_tma && !a.y_f32 && slab_bytes <= stages * stage_bytes) ? 1 : 0;
  g.BN = BN;
  g.stages = stages;
  g.status = a.status;
  const bool split = a.k_splits > 1;
  if (split && (BITS != 0 || !a.y_f32 || a.kb_per_split < 1 ||
                static_cast<int64_t>(a.k_splits - 1) * a.kb_per_split >= (a.K + kBK - 1) / kBK))
    return cudaErrorInvalidValue;   // every split must own at least one main K block
  g.kb_per_split = split ? a.kb_per_split : 0;
  g.split_stride = split ? a.split_stride : 0;
  if (split) g.y_tma = 0;
  const dim3 grid(static_cast<unsigned>((a.M + BM - 1) / BM),
                  static_cast<unsigned>((a.T + BN - 1) / BN),
                  static_cast<unsigned>(split ? a.k_splits : 1));
  return launch_kernel(ttq_gemm_kernel<BITS, BM, TC>, grid, dim3(cta_threads<BM>()), smem, stream,
                       pdl, maps.a0, maps.b0, maps.a1, maps.b1, maps.c0, maps.y, g);
}

template <int BITS>
cudaError_t launch_bits(const GemmArgs& a, const GemmMaps& maps, int BN, int BM,
                        cudaStream_t stream, bool pdl) {
  if (BITS == 0) {
    if (BM == 256) return launch_tile<BITS, 256, false>(a, maps, BN, stream, pdl);
    return launch_tile<BITS, 128, false>(a, maps, BN, stream, pdl);
  }
  if (a.codes_tma) {
    if (BM == 256) return launch_tile<BITS, 256, true>(a, maps, BN, stream, pdl);
    return launch_tile<BITS, 128, true>(a, maps, BN, stream, pdl);
  }
  if (BM == 256) return launch_tile<BITS, 256, false>(a, maps, BN, stream, pdl);
  return launch_tile<BITS, 128, false>(a, maps, BN, stream, pdl);
}

// AX[t][k] = bf16(sum over s of P[s][t][k]), the splits added in order.
__global__ void ax_reduce_kernel(const float* __restrict__ P, int splits, int64_t T, int64_t r,
                                 __nv_bfloat16* __restrict__ AX, int64_t ax_ld) {
  allow_dependents_launch();
  grid_dependency_wait();
  const int64_t n = T * r;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += __ldcg(P + s * n + i);
    const int64_t t = i / r;
    AX[t * ax_ld + (i - t * r)] = __float2bfloat16_rn(acc);
  }
}

// Y[i] = the sum over s of P[s][i], the splits added in order and the sum
// rounded once (to bf16, or kept in float32); n = T * ldy elements.
__global__ void y_reduce_kernel(const float* __restrict__ P, int splits, int64_t n,
                                void* __restrict__ Y, int y_f32) {
  allow_dependents_launch();
  grid_dependency_wait();   // the partials come from the previous kernel
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n % 4 == 0) {
    const int64_t nv = n / 4;
    for (int64_t i = i0; i < nv; i += stride) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < splits; ++s) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(P + s * n) + i);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      if (y_f32) {
        reinterpret_cast<float4*>(Y)[i] = acc;
      } else {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 u;
        memcpy(&u.x, &lo, 4);
        memcpy(&u.y, &hi, 4);
        reinterpret_cast<uint2*>(Y)[i] = u;
      }
    }
  } else {
    for (int64_t i = i0; i < n; i += stride) {
      float acc = 0.f;
      for (int s = 0; s < splits; ++s) acc += __ldcs(P + s * n + i);
      if (y_f32) static_cast<float*>(Y)[i] = acc;
      else static_cast<__nv_bfloat16*>(Y)[i] = __float2bfloat16_rn(acc);
    }
  }
}

}  // namespace

AxSplit ax_split_plan(int64_t r, int64_t T, int64_t d, int num_sms) {
  const int64_t kb = (d + kBK - 1) / kBK;
  const int64_t tiles = ((r + 127) / 128) * ((T + gemm_block_n(T) - 1) / gemm_block_n(T));
  int64_t s = tiles > 0 ? num_sms / tiles : 1;
  if (s > kb / 4) s = kb / 4;
  if (s < 2) return {1, static_cast<int>(kb)};
  const int64_t per = (kb + s - 1) / s;
  return {static_cast<int>((kb + per - 1) / per), static_cast<int>(per)};
}

cudaError_t launch_ax_reduce(const float* P, int splits, int64_t T, int64_t r, void* AX,
                             int64_t ax_ld, cudaStream_t stream, bool pdl) {
  const int64_t n = T * r;
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  return launch_kernel(ax_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                       pdl, P, splits, T, r, static_cast<__nv_bfloat16*>(AX), ax_ld);
}

int gemm_code_tile_words(int bits) { return bits == 2 ? 4 : 8; }

int gemm_block_n(int64_t T) {
  if (T >= 256) return 256;
  int64_t bn = (T + 15) / 16 * 16;
  if (bn < 16) bn = 16;
  return static_cast<int>(bn);
}

void gemm_tile_shape(int bits, int64_t M, int64_t T, int num_sms, int* block_m, int* block_n) {
  // Cost of a shape: waves of CTAs times the time of one CTA, taken as
  // proportional to (BN + 24) (24: the fixed prologue / epilogue share) and
  // to 2.0 for 256-row tiles, 1.4 for 128-row tiles (which move twice the X
  // bytes per FLOP).  With codes, the dequantisation of a K block takes
  // about as long as 256 tokens of MMA whatever BN is, so BN counts as at
  // least 256 there.  256-row tiles need M > 128.
  const int64_t bn_max = T >= 256 ? 256 : (T + 15) / 16 * 16;
  double best = 0.0;
  int best_m = 128, best_n = 16;
  for (int bm = 256; bm >= 128; bm -= 128) {
    if (bm == 256 && M <= 128) continue;
    for (int bn = static_cast<int>(bn_max); bn >= 16; bn -= 16) {
      const int64_t tiles = (M + bm - 1) / bm * ((T + bn - 1) / bn);
      const int64_t waves = (tiles + num_sms - 1) / num_sms;
      const int work = bits != 0 && bn < 256 ? 256 : bn;
      const double cost = static_cast<double>(waves) * (bm == 256 ? 2.0 : 1.4) * (work + 24);
      if (best == 0.0 || cost < best) {
        best = cost;
        best_m = bm;
        best_n = bn;
      }
    }
  }
  *block_m = best_m;
  *block_n = best_n;
}

GemmPlan gemm_plan_plain(int64_t M, int64_t T, int64_t K, int64_t K_tail, int num_sms,
                         bool allow_split) {
  // Unsplit, the tile shape is gemm_tile_shape's.  A K split is weighed
  // against it with a time model: the larger of
  //  - the tensor-core time: waves x K blocks per CTA x 4 BN (BM = 256) or
  //    2 BN (BM = 128) cycles (4096 multiply-adds per SM and cycle), at the
  //    power-capped clock of about 1.7 GHz;
  //  - the time to bring the operand tiles from L2 into shared memory: each
  //    CTA reads (BM + BN) x 128 bytes per K block, at about 12 TB/s over the
  //    device and at most 128 bytes per cycle into one SM;
  // plus, with K split in s parts, the float32 partial sums written and read
  // once more and Y written (about 6 TB/s), and the reduction's launch.  The
  // unsplit product at 4096 x 4096 x 2048 (256 x 240 tiles) and at
  // 4096 x 512 x 11008 (256 x 64 tiles), measured on B200, is bound by the
  // L2 term: 48.6 and 93 us against 48.8 and 75.6 us modelled.  (As a choice
  // among unsplit shapes the model misleads: it prefers 256 x 256 tiles,
  // which measured 2-4% slower than gemm_tile_shape's at 4096 x 4096 x 2048
  // and 28672 x 1024 x 8192.)  A split is taken when the model puts it 10%
  // ahead of the unsplit shape.
  constexpr double kClock = 1.7e9, kL2 = 12e12, kSmL2 = 128.0 * kClock, kHbm = 6e12;
  constexpr double kLaunch = 2e-6;
  constexpr int kMaxSplits = 8, kMinBlocksPerSplit = 8;
  const int64_t kb = (K + kBK - 1) / kBK;
  const int64_t kbt = (K_tail + kBK - 1) / kBK;
  auto model = [&](int bm, int bn, int64_t s, int64_t per) {
    const int64_t tiles = (M + bm - 1) / bm * ((T + bn - 1) / bn);
    const int64_t ctas = tiles * s;
    const int64_t waves = (ctas + num_sms - 1) / num_sms;
    const int64_t kcta = per + kbt;   // the last split's blocks, tail included
    const double t_mma = static_cast<double>(waves * kcta) * (bm == 256 ? 4.0 : 2.0) * bn / kClock;
    const double bytes = static_cast<double>(bm + bn) * 128.0 * static_cast<double>(kcta);
    const double t_l2 = std::max(static_cast<double>(ctas) * bytes / kL2,
                                 static_cast<double>(waves) * bytes / kSmL2);
    const double t_red =
        s > 1 ? static_cast<double>(2 * s + 1) * static_cast<double>(T * M) * 4.0 / kHbm + kLaunch
              : 0.0;
    return std::max(t_mma, t_l2) + t_red;
  };
  GemmPlan plan{128, 16, 1, 0};
  gemm_tile_shape(0, M, T, num_sms, &plan.block_m, &plan.block_n);
  if (!allow_split) return plan;
  const double t1 = model(plan.block_m, plan.block_n, 1, kb);
  double ts = -1.0;
  GemmPlan split = plan;
  const int64_t bn_max = T >= 256 ? 256 : (T + 15) / 16 * 16;
  for (int bm = 256; bm >= 128; bm -= 128) {
    if (bm == 256 && M <= 128) continue;
    for (int bn = static_cast<int>(bn_max); bn >= 16; bn -= 16) {
      for (int64_t s = 2; s <= kMaxSplits && kb / s >= kMinBlocksPerSplit; ++s) {
        const int64_t per = (kb + s - 1) / s;
        if ((kb + per - 1) / per != s) continue;   // another s gives these splits
        const double t = model(bm, bn, s, per);
        if (ts < 0.0 || t < ts) {
          ts = t;
          split = GemmPlan{bm, bn, static_cast<int>(s), static_cast<int>(per)};
        }
      }
    }
  }
  return ts >= 0.0 && ts < 0.9 * t1 ? split : plan;
}

cudaError_t launch_y_reduce(const float* P, int splits, int64_t n, void* Y, bool y_f32,
                            cudaStream_t stream, bool pdl) {
  if (n == 0) return cudaSuccess;
  const int64_t work = n % 4 == 0 ? n / 4 : n;
  int64_t blocks = (work + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  return launch_kernel(y_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                       pdl, P, splits, n, Y, y_f32 ? 1 : 0);
}

cudaError_t launch_dequant_gemm(const GemmArgs& args, const GemmMaps& maps, int block_n,
                                int block_m, cudaStream_t stream, bool pdl) {
  if (args.M == 0 || args.T == 0) return cudaSuccess;
  if (block_n % 16 != 0 || block_n < 16 || block_n > 256) return cudaErrorInvalidValue;
  if (block_m != 128 && block_m != 256) return cudaErrorInvalidValue;
  switch (args.bits) {
    case 0:
      return launch_bits<0>(args, maps, block_n, block_m, stream, pdl);
    case 2:
      return launch_bits<2>(args, maps, block_n, block_m, stream, pdl);
    case 3:
      return launch_bits<3>(args, maps, block_n, block_m, stream, pdl);
    case 4:
      return launch_bits<4>(args, maps, block_n, block_m, stream, pdl);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ttq
