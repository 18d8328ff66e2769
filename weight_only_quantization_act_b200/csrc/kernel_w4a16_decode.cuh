// kernel_w4a16_decode.cuh - the deployment GEMM of an AWQ-quantized linear for few tokens (decode, small
// batches): Y = X' deq(W)^T with M <= 64 tokens. At this size the work is reading and unpacking the packed
// weights, so the weight rows take the MMA's M side, the groups are split into slices until every SM has
// a share, and the per-weight arithmetic is moved off the CUDA cores:
//
//   deq(W)[o, k] = (q - z_g) * step_g for the group g of 128 in-features holding k, so
//   Y[m, o] = sum_g step_g * ( S_g[o, m] - (128 + z_g) * Sx_g[m] ),
//   S_g[o, m] = sum_{k in g} (128 + q[o, k]) * x'[m, k],   Sx_g[m] = sum_{k in g} x'[m, k].
//
// The tensor cores compute S_g from bf16 operands (128 + q is the bf16 pattern 0x4300 | q, an OR with the
// code nibble, and every product of two bf16 values is exact in the fp32 accumulator), one group per
// accumulator; the CUDA cores then apply the group's step and zero point once per output element and
// group instead of once per weight. The weights thus enter with their exact dequantized value
// (q - z) * step ("GPU 硬件级反量化算子内联融合" on the bjdmk.com.cn AWQ article: unpack with shifts and
// masks, convert, apply the group scale and offset; here the scale and offset are applied after the
// products of each group).
//
// Nibble order. A code word holds in-features 8c .. 8c+7 in nibbles 0..7. One AND-OR per register turns
// the word shifted right by 4j into the bf16 pair (128 + q_j, 128 + q_{j+4}), so the operand row holds
// each word's in-features in the order 0 4 1 5 2 6 3 7. X' is permuted the same way inside every 16-byte
// chunk (8 in-features), which leaves the products and sums unchanged. A small kernel before this one
// writes that permuted copy of X' (nt rows, zero past M) and every Sx_g once, instead of every CTA
// redoing them; it lets this kernel start early (programmatic dependent launch), and only the loader
// waits for it, after requesting its first code boxes.
//
// CTA (b, c) covers weight rows [128 b, 128 b + 128) and groups [c * gp, (c + 1) * gp) (gp even). The
// unpacked operand of a group (128 rows x 128 in-features) lives in tensor memory (tcgen05.mma reads A
// from there), three groups at a time, next to the accumulators. Warps:
//   0      loads: one TMA box of code words per two groups [128 rows x 32 words] (128-byte swizzle),
//          X' per group as two [nt x 64] boxes (128-byte swizzle) and Sx_g (one bulk copy), each into a
//          ring of its own
//   1      tensor memory; one thread issues the 8 MMAs of a group (M = 128, N = nt, K = 16)
//   2-9    unpack: warps 2-5 take the even groups, warps 6-9 the odd ones; lane l of warp w unpacks row
//          32 (w % 4) + l (the tensor-memory lanes warp w may write) with two 32-column stores
//   10-13  per group: S_g of their lane quarter, minus the zero-point term, times step, added to per-row
//          registers (steps and zero points read from global memory four groups ahead); at the end Y, or
//          this slice's partial sums
// With several slices the last CTA of a row block to finish (a per-block counter it resets to zero)
// adds the slices' partial sums in slice order (deterministic). All waits are bounded; a timeout is
// recorded in the caller's status word.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "numerics.cuh"
#include "ptx.cuh"

namespace awq {
namespace dec {

constexpr int ROWS = 128;                     // weight rows per CTA (the MMA's M)
constexpr int BK = 64;                        // in-features per k-block (one 128-byte swizzle row)
constexpr int GK = 128;                       // in-features per group
constexpr int UK = 16;                        // K of one MMA
constexpr int MAX_NT = 64;                    // tokens per launch (the MMA's N, a multiple of 16)
constexpr int GROUPS_PER_BOX = 2;             // code box: 32 words = 128 bytes per row = 2 groups
constexpr int C_BYTES = ROWS * 128;           // 16 KB
constexpr int A_COLS = GK / 2;                // tensor-memory columns of one group's operand (64)
constexpr int UNPACK_WARPS = 8;
constexpr int EPI_WARP0 = 2 + UNPACK_WARPS;   // warps 10-13
constexpr int THREADS = 32 * (EPI_WARP0 + 4);  // 448
constexpr int MAX_SLICES = 16;
constexpr int SX_STAGES = 8;                  // Sx_g of the groups in flight between loader and epilogue
constexpr int SZ_AHEAD = 4;                   // groups of steps and zero points an epilogue thread has in flight

template <int NT>
struct Shape {
  static constexpr int CTAS_PER_SM = NT <= 16 ? 2 : 1;
  static constexpr int C_STAGES = 3;                                    // code boxes in flight
  static constexpr int X_BYTES = 2 * NT * 128;                          // one group: two [NT x 64] tiles
  static constexpr int X_STAGES = NT <= 16 ? 8 : (96 * 1024) / X_BYTES; // X' groups in flight
  static constexpr int ACC_STAGES = 4;                                  // group accumulators S_g
  static constexpr int A_BUFS = 3;                                      // group operands in flight
  static constexpr int A_COL0 = ACC_STAGES * NT;
  static constexpr int USED_COLS = A_COL0 + A_BUFS * A_COLS;
  static constexpr uint32_t TMEM_COLS = USED_COLS <= 128 ? 128 : (USED_COLS <= 256 ? 256 : 512);
  static constexpr int SMEM = C_STAGES * C_BYTES + X_STAGES * X_BYTES + SX_STAGES * NT * 4 + 1024;
};
static_assert(Shape<16>::USED_COLS <= 256 && Shape<16>::SMEM <= 113 * 1024, "two CTAs per SM");
static_assert(Shape<64>::USED_COLS <= 512, "tensor memory");
static_assert(Shape<64>::SMEM <= 227 * 1024 && Shape<48>::SMEM <= 227 * 1024, "one CTA per SM");

// Slices of the groups per row block the workspace is sized for: enough for 512 CTAs, at most
// MAX_SLICES. The workspace holds partial[n_rb][slices][MAX_NT][ROWS] fp32 and one counter per row block.
__host__ __device__ constexpr int64_t max_slices(int64_t n_rb) {
  return n_rb >= 512 ? 1 : ((512 + n_rb - 1) / n_rb < MAX_SLICES ? (512 + n_rb - 1) / n_rb : MAX_SLICES);
}

enum : unsigned int {
  kSiteDecodeEmpty = 20,
  kSiteDecodeFull = 21,
  kSiteDecodeDequant = 22,
  kSiteDecodeAcc = 23,
};

struct Params {
  const float* steps;     // [O][G]
  const float* zeros;     // [O][G]
  __nv_bfloat16* Y;       // [M][ldy]
  float* partial;         // [n_rb][slices][nt][ROWS]
  unsigned int* counter;  // [n_rb], zero at launch and left zero
  const float* sx;        // [G][nt] group sums of X' (decode_prep_kernel)
  int64_t M, O, G, ldy;
  int num_groups;         // K / 128
  int g_per;              // groups per slice, even
  int slices;
  uint32_t idesc;
  DeviceStatus* status;
  uint64_t limit_ns;
};

// Bounded wait by one thread; records a timeout (never reads the status, so a stale word from an earlier
// call cannot cut this one short).
// The waits let the hardware suspend the waiting threads (up to 20 us per try) instead of spinning, so
// waiting warps take few issue slots from the unpack warps.
constexpr uint32_t kSleepNs = 20000;

__device__ __forceinline__ bool wait_thread(uint32_t bar, uint32_t parity, const Params& p, unsigned int where) {
  if (mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
  const uint64_t t0 = global_timer_ns();
#pragma unroll 1
  while (!mbar_try_wait_sleep(bar, parity, kSleepNs))
    if (global_timer_ns() - t0 > p.limit_ns) {
      raise_timeout(p.status, where);
      return false;
    }
  return true;
}

// Warp-uniform bounded wait: every lane polls, the warp leaves together.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const Params& p, unsigned int where) {
  // the phase has usually completed already: one poll before the timer is read
  if (__all_sync(0xffffffffu, mbar_try_wait_sleep(bar, parity, kSleepNs))) return true;
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
  if (lane == 0) t0 = global_timer_ns();
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait_sleep(bar, parity, kSleepNs))) return true;
    int give_up = 0;
    if (lane == 0 && global_timer_ns() - t0 > p.limit_ns) {
      raise_timeout(p.status, where);
      give_up = 1;
    }
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
  }
}

__device__ __forceinline__ void epilogue_sync() {  // warps 10-13 only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}

// (128 + q) as bf16 pairs from a code word: register j holds the nibbles j and j + 4 (in-features 8c + j and
// 8c + j + 4 of word c) in its low and high half, 0x4300 | q each. The word shifted right by 4 j (a
// multiply-high by 2^(32 - 4 j), which runs on the FMA pipe and leaves the ALU pipe to the AND-ORs)
// brings both nibbles to bits 0-3 and 16-19.
__device__ __forceinline__ uint32_t nibble_pair_bf16(uint32_t w_shifted) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w_shifted));  // (a & b) | c
  return r;
}
__device__ __forceinline__ uint32_t shr_fma(uint32_t w, uint32_t pow2) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(pow2));
  return r;
}
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&v)[4]) {
  v[0] = nibble_pair_bf16(w);
  v[1] = nibble_pair_bf16(shr_fma(w, 1u << 28));
  v[2] = nibble_pair_bf16(shr_fma(w, 1u << 24));
  v[3] = nibble_pair_bf16(shr_fma(w, 1u << 20));
}

// X' for the few-token kernel: Xp[m][k] = X[m][k] for m < M, zero for M <= m < nt, with each 16-byte chunk
// of 8 in-features in the operand order 0 4 1 5 2 6 3 7; Sx[g][m] = the sum of X[m][k] over the group's
// 128 in-features (fp32: each chunk's 8 values in increasing k, then the 16 chunk sums in order; zero past
// M). One CTA per group; every (token, chunk) pair is one 16-byte load, so the kernel is one memory round
// trip long.
constexpr int PREP_THREADS = 128;
__global__ void __launch_bounds__(PREP_THREADS) decode_prep_kernel(const uint16_t* __restrict__ X, int64_t M,
                                                                   int64_t K, int64_t ldx, int nt,
                                                                   uint16_t* __restrict__ Xp, float* __restrict__ Sx) {
  pdl_launch_dependents();
  __shared__ float chunk_sum[MAX_NT][GK / 8];
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * GK;
  for (int task = threadIdx.x; task < nt * (GK / 8); task += PREP_THREADS) {
    const int m = task / (GK / 8), ch = task % (GK / 8);
    const uint4 v = m < M ? *reinterpret_cast<const uint4*>(X + m * ldx + k0 + 8 * ch) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(Xp + static_cast<int64_t>(m) * K + k0 + 8 * ch) =
        make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632), __byte_perm(v.y, v.w, 0x5410),
                   __byte_perm(v.y, v.w, 0x7632));
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      sum = __fadd_rn(__fadd_rn(sum, __uint_as_float(e[k] << 16)), __uint_as_float(e[k] & 0xFFFF0000u));
    chunk_sum[m][ch] = sum;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    const int m = threadIdx.x;
    float sum = 0.0f;
#pragma unroll
    for (int ch = 0; ch < GK / 8; ++ch) sum = __fadd_rn(sum, chunk_sum[m][ch]);
    Sx[static_cast<int64_t>(blockIdx.x) * nt + m] = sum;
  }
}

template <int NT>
__global__ void __launch_bounds__(THREADS, Shape<NT>::CTAS_PER_SM)
    w4a16_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC, Params p) {
  // tmX covers the permuted copy Xp [nt][K]; p.sx holds Sx [G][nt] (both from decode_prep_kernel)
  using S = Shape<NT>;
  constexpr int CS = S::C_STAGES, XS = S::X_STAGES, AS = S::ACC_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int AB = S::A_BUFS;
  __shared__ __align__(8) uint64_t bars[2 * CS + 2 * XS + 2 * AB + 2 * AS + 2 * SX_STAGES];
  __shared__ uint32_t tmem_slot;
  __shared__ int failed;
  __shared__ unsigned int ticket;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = static_cast<int>(blockIdx.x) / p.slices;
  const int slice = static_cast<int>(blockIdx.x) - rb * p.slices;
  const int64_t row0 = static_cast<int64_t>(rb) * ROWS;
  const int g0 = slice * p.g_per;
  const int ng = max(0, min(p.g_per, p.num_groups - g0));

  const uint32_t bar0 = smem_u32(&bars[0]);
  auto cfull_bar = [&](int c) { return bar0 + 8u * c; };                          // codes landed
  auto cempty_bar = [&](int c) { return bar0 + 8u * (CS + c); };                  // codes read
  auto xfull_bar = [&](int x) { return bar0 + 8u * (2 * CS + x); };               // X' landed
  auto xempty_bar = [&](int x) { return bar0 + 8u * (2 * CS + XS + x); };         // MMAs done with X'
  auto dq_bar = [&](int a) { return bar0 + 8u * (2 * CS + 2 * XS + a); };         // operand a written
  auto afree_bar = [&](int a) { return bar0 + 8u * (2 * CS + 2 * XS + AB + a); };  // MMAs done with it
  auto accfull_bar = [&](int s) { return bar0 + 8u * (2 * CS + 2 * XS + 2 * AB + s); };
  auto accempty_bar = [&](int s) { return bar0 + 8u * (2 * CS + 2 * XS + 2 * AB + AS + s); };
  auto sxfull_bar = [&](int t) { return bar0 + 8u * (2 * CS + 2 * XS + 2 * AB + 2 * AS + t); };
  auto sxempty_bar = [&](int t) { return bar0 + 8u * (2 * CS + 2 * XS + 2 * AB + 2 * AS + SX_STAGES + t); };
  const uint32_t base = smem_u32(smem);
  auto c_tile = [&](int c) { return base + static_cast<uint32_t>(c) * C_BYTES; };
  auto x_tile = [&](int x, int h) {  // half h (in-features 64 h .. 64 h + 63 of the group)
    return base + CS * C_BYTES + static_cast<uint32_t>(x) * S::X_BYTES + static_cast<uint32_t>(h * NT * 128);
  };
  auto sx_slot = [&](int t) {  // Sx_g[NT] fp32
    return base + CS * C_BYTES + XS * S::X_BYTES + static_cast<uint32_t>(t * NT * 4);
  };

  if (threadIdx.x == 0) {
    for (int c = 0; c < CS; ++c) {
      mbar_init(cfull_bar(c), 1);
      mbar_init(cempty_bar(c), UNPACK_WARPS);  // each warp reads one of the box's two groups
    }
    for (int x = 0; x < XS; ++x) {
      mbar_init(xfull_bar(x), 1);
      mbar_init(xempty_bar(x), 1);
    }
    for (int a = 0; a < AB; ++a) {
      mbar_init(dq_bar(a), UNPACK_WARPS / 2);  // the four warps of the set that writes the group
      mbar_init(afree_bar(a), 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(accfull_bar(s), 1);
      mbar_init(accempty_bar(s), 4);
    }
    for (int t = 0; t < SX_STAGES; ++t) {
      mbar_init(sxfull_bar(t), 1);  // the loader's arrive with the bulk copy's bytes
      mbar_init(sxempty_bar(t), 4);
    }
    failed = 0;
    ticket = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
  }
  // Loads of local group i: its code box when i is even (the box holds groups i and i + 1) and X'.
  // Warp 0 only, all lanes; false when a wait gave up.
  auto load_codes = [&](int i) -> bool {
    const int j = i / GROUPS_PER_BOX;
    const int c = j % CS;
    const uint32_t use = static_cast<uint32_t>(j / CS);
    if (use > 0 && !wait_warp(cempty_bar(c), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(cfull_bar(c), C_BYTES);
      tma_load_2d(c_tile(c), &tmC, (g0 + i) * (GK / 8), static_cast<int32_t>(row0), cfull_bar(c));
    }
    __syncwarp();
    return true;
  };
  // X' of local group i, and its Sx_g into the Sx ring (freed by the epilogue).
  auto load_x = [&](int i) -> bool {
    const int x = i % XS, t = i % SX_STAGES;
    const uint32_t use = static_cast<uint32_t>(i / XS), sx_use = static_cast<uint32_t>(i / SX_STAGES);
    if (use > 0 && !wait_warp(xempty_bar(x), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (sx_use > 0 && !wait_warp(sxempty_bar(t), (sx_use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(xfull_bar(x), S::X_BYTES);
      tma_load_2d(x_tile(x, 0), &tmX, (g0 + i) * GK, 0, xfull_bar(x));
      tma_load_2d(x_tile(x, 1), &tmX, (g0 + i) * GK + BK, 0, xfull_bar(x));
      mbar_arrive_expect_tx(sxfull_bar(t), NT * 4);
      bulk_load(sx_slot(t), p.sx + static_cast<int64_t>(g0 + i) * NT, NT * 4, sxfull_bar(t));
    }
    __syncwarp();
    return true;
  };
  // The first groups need no free slots: warp 0 requests them right after initialising the barriers, so
  // the first memory round trip overlaps the tensor-memory allocation and the CTA barrier.
  const int pre_c = min(ng, CS * GROUPS_PER_BOX);
  const int pre_x = min(ng, min(XS, SX_STAGES));
  if (warp == 0) {
    __syncwarp();  // the barriers thread 0 initialised are visible to the whole warp
    // the code boxes first (they do not depend on the kernel before this one), then, once its X' copy
    // and group sums are complete, X' and Sx of the first groups
    for (int i = 0; i < pre_c; i += GROUPS_PER_BOX) load_codes(i);
    pdl_wait();
    for (int i = 0; i < pre_x; ++i) load_x(i);
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------------------ loads
    // Both rings are refilled in group order: a code box once its slot is free (the box CS boxes
    // earlier unpacked), X' once its slot is (the MMAs XS groups earlier done).
    for (int i = 0; i < ng; ++i) {
      bool ok = true;
      if (i >= pre_c && i % GROUPS_PER_BOX == 0) ok = load_codes(i);
      if (ok && i >= pre_x) ok = load_x(i);
      if (!ok) {
        failed = 1;
        break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ MMA
    if (elect_one()) {
      bool ok = true;
      for (int i = 0; i < ng && ok; ++i) {
        const int x = i % XS, s = i % AS, a = i % AB;
        const uint32_t acc_use = static_cast<uint32_t>(i / AS);
        if (!wait_thread(xfull_bar(x), static_cast<uint32_t>(i / XS) & 1u, p, kSiteDecodeFull) ||
            !wait_thread(dq_bar(a), static_cast<uint32_t>(i / AB) & 1u, p, kSiteDecodeDequant) ||
            (acc_use > 0 && !wait_thread(accempty_bar(s), (acc_use - 1u) & 1u, p, kSiteDecodeAcc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(s * NT);
        const uint32_t at = tmem_base + static_cast<uint32_t>(S::A_COL0 + a * A_COLS);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            umma_bf16_ts(d, at + static_cast<uint32_t>((h * (BK / UK) + kk) * (UK / 2)),
                         smem_desc_sw128(x_tile(x, h) + kk * UK * 2), p.idesc, (h | kk) != 0 ? 1u : 0u);
        umma_commit(afree_bar(a));
        umma_commit(xempty_bar(x));
        umma_commit(accfull_bar(s));
      }
      if (!ok) failed = 1;
    }
    __syncwarp();
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------------------------ unpack
    // Warps 2-5 take the even groups, 6-9 the odd ones; group i goes to operand buffer i % 3.
    const int q = warp & 3, set = (warp - 2) >> 2;
    const int r = 32 * q + lane;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    for (int i = set; i < ng; i += 2) {
      const int j = i / GROUPS_PER_BOX, c = j % CS;
      if (!wait_warp(cfull_bar(c), static_cast<uint32_t>(j / CS) & 1u, p, kSiteDecodeFull)) {
        failed = 1;
        break;
      }
      // words 16 (i % 2) .. + 15 of row r: 16-byte chunks 4 (i % 2) .. + 3 of its swizzled line
      const uint32_t line_c = c_tile(c) + static_cast<uint32_t>(r) * 128u;
      uint4 wv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        wv[u] = ld_shared_v4(line_c + (((static_cast<uint32_t>(4 * (i % GROUPS_PER_BOX) + u)) ^ sw) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(cempty_bar(c));  // the words are in registers
      // the operand
      const int a = i % AB;
      const uint32_t ause = static_cast<uint32_t>(i / AB);
      if (ause > 0 && !wait_warp(afree_bar(a), (ause - 1u) & 1u, p, kSiteDecodeEmpty)) {
        failed = 1;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w[8] = {wv[2 * h].x, wv[2 * h].y, wv[2 * h].z, wv[2 * h].w,
                               wv[2 * h + 1].x, wv[2 * h + 1].y, wv[2 * h + 1].z, wv[2 * h + 1].w};
        uint32_t v[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t v4[4];
          unpack_word(w[u], v4);
#pragma unroll
          for (int k = 0; k < 4; ++k) v[4 * u + k] = v4[k];
        }
        tmem_st32(tl + static_cast<uint32_t>(S::A_COL0 + a * A_COLS + h * (A_COLS / 2)), v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_bar(a));
    }
  } else {
    // ------------------------------------------------------------------------------ group epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    const int r = 32 * q + lane;
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const int64_t o_ld = min(row0 + r, p.O - 1);  // rows past O: any valid address (results dropped)
    const float* st_row = p.steps + o_ld * p.G + g0;
    const float* z_row = p.zeros + o_ld * p.G + g0;
    float y[NT];
#pragma unroll
    for (int m = 0; m < NT; ++m) y[m] = 0.0f;
    // steps and zero points SZ_AHEAD groups ahead, in registers
    float st_n[SZ_AHEAD], z_n[SZ_AHEAD];
#pragma unroll
    for (int u = 0; u < SZ_AHEAD; ++u) {
      st_n[u] = u < ng ? __ldg(st_row + u) : 0.0f;
      z_n[u] = u < ng ? __ldg(z_row + u) : 0.0f;
    }
    bool have = true;
    for (int i = 0; i < ng; ++i) {
      const int s = i % AS, t = i % SX_STAGES;
      const float step = st_n[0];
      const float c = __fadd_rn(128.0f, z_n[0]);
#pragma unroll
      for (int u = 0; u + 1 < SZ_AHEAD; ++u) {
        st_n[u] = st_n[u + 1];
        z_n[u] = z_n[u + 1];
      }
      st_n[SZ_AHEAD - 1] = i + SZ_AHEAD < ng ? __ldg(st_row + i + SZ_AHEAD) : 0.0f;
      z_n[SZ_AHEAD - 1] = i + SZ_AHEAD < ng ? __ldg(z_row + i + SZ_AHEAD) : 0.0f;
      if (!wait_warp(accfull_bar(s), static_cast<uint32_t>(i / AS) & 1u, p, kSiteDecodeAcc) ||
          !wait_warp(sxfull_bar(t), static_cast<uint32_t>(i / SX_STAGES) & 1u, p, kSiteDecodeAcc)) {
        have = false;
        break;
      }
      tc_fence_after();
      // 16 columns at a time: y[m] += step * (S_g[r, m] - (128 + z) * Sx_g[m])
#pragma unroll
      for (int cc = 0; cc < NT / 16; ++cc) {
        float sg[16];
        tmem_ld16(tlane + static_cast<uint32_t>(s * NT + 16 * cc), sg);
#pragma unroll
        for (int k4 = 0; k4 < 16; k4 += 4) {
          float4 xs;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(xs.x), "=f"(xs.y), "=f"(xs.z), "=f"(xs.w)
                       : "r"(sx_slot(t) + 4u * static_cast<uint32_t>(16 * cc + k4))
                       : "memory");
          // paired fp32: t = S - c * Sx, y = y + step * t, two tokens per instruction
#pragma unroll
          for (int k = 0; k < 4; k += 2) {
            const int m = 16 * cc + k4 + k;
            const uint64_t t = fx2_fma(fx2(-c, -c), fx2(k == 0 ? xs.x : xs.z, k == 0 ? xs.y : xs.w),
                                       fx2(sg[k4 + k], sg[k4 + k + 1]));
            fx2_split(fx2_fma(fx2(step, step), t, fx2(y[m], y[m + 1])), y[m], y[m + 1]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(accempty_bar(s));
        mbar_arrive(sxempty_bar(t));
      }
    }
    if (!have) failed = 1;
    if (p.slices == 1) {
      // One slice: the sums are the result; lane r writes row r of every token (coalesced per token).
      const int64_t o = row0 + r;
#pragma unroll
      for (int m = 0; m < NT; ++m)
        if (m < p.M && o < p.O) p.Y[m * p.ldy + o] = __float2bfloat16_rn(have ? y[m] : 0.0f);
    } else {
      // Slice `slice` of the row block's partial sums, then a ticket.
      float* mine = p.partial + (static_cast<int64_t>(rb) * p.slices + slice) * NT * ROWS + r;
#pragma unroll
      for (int m = 0; m < NT; ++m) __stcg(mine + m * ROWS, have ? y[m] : 0.0f);
      __threadfence();
      epilogue_sync();
      if (warp == EPI_WARP0 && lane == 0) {
        // Every CTA takes a ticket, even after a timeout, and the last one hands the counter back at
        // zero, so the next call needs no clearing.
        ticket = atomicAdd(p.counter + rb, 1u);
        if (ticket == static_cast<unsigned int>(p.slices - 1)) p.counter[rb] = 0u;
      }
    }
  }

  __syncwarp();
  __syncthreads();
  if (p.slices > 1 && ticket == static_cast<unsigned int>(p.slices - 1)) {
    // Last slice of this row block: every other slice's sums are visible (each CTA fenced before taking
    // its ticket). The whole CTA adds them in slice order, four rows per item.
    __threadfence();
    const float* blk = p.partial + static_cast<int64_t>(rb) * p.slices * NT * ROWS;
    const int items = static_cast<int>(p.M) * (ROWS / 4);
    // One item per thread per pass and eight slices per round, so eight loads are in flight at once.
    for (int it = static_cast<int>(threadIdx.x); it < items; it += THREADS) {
      const int t = it / (ROWS / 4);
      const int r4 = (it - t * (ROWS / 4)) * 4;
      if (row0 + r4 >= p.O) continue;  // O % 8 == 0: four rows are all in or all out
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 1
      for (int c0 = 0; c0 < p.slices; c0 += 8) {
        float4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          v[c] = c0 + c < p.slices
                     ? __ldcg(reinterpret_cast<const float4*>(blk + (static_cast<int64_t>(c0 + c) * NT + t) * ROWS + r4))
                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c0 + c >= p.slices) continue;
          if (c0 + c == 0) {
            acc = v[0];  // slice order: ((s0 + s1) + s2) + ...
          } else {
            acc.x = __fadd_rn(acc.x, v[c].x);
            acc.y = __fadd_rn(acc.y, v[c].y);
            acc.z = __fadd_rn(acc.z, v[c].z);
            acc.w = __fadd_rn(acc.w, v[c].w);
          }
        }
      }
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      *reinterpret_cast<uint2*>(p.Y + t * p.ldy + row0 + r4) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
  if (failed) {  // let copies still in flight land before the shared memory is given up
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace dec
}  // namespace awq
