// kernel_w4a16_decode.cuh - the deployment GEMM of an AWQ-quantized linear for few tokens (decode, small
// batches): Y = X' deq(W)^T with M <= 64 tokens. At this size the work is reading and unpacking the packed
// weights, so the weight rows take the MMA's M side, the k-blocks are split until every SM has a share,
// and the per-weight arithmetic is moved off the CUDA cores:
//
//   deq(W)[o, k] = (q - z_g) * step_g for the group g of 128 in-features holding k, so
//   Y[m, o] = sum_g step_g * ( S_g[o, m] - (128 + z_g) * Sx_g[m] ),
//   S_g[o, m] = sum_{k in g} (128 + q[o, k]) * x'[m, k],   Sx_g[m] = sum_{k in g} x'[m, k].
//
// The tensor cores compute S_g exactly from bf16 operands (128 + q is the bf16 pattern 0x4300 | q, an
// OR with the code nibble, and every product of two bf16 values is exact in the fp32 accumulator), one
// group per accumulator; the CUDA cores then apply the group's step and zero point once per output
// element and group instead of once per weight. The weights thus enter with their exact dequantized
// value (q - z) * step ("GPU 硬件级反量化算子内联融合" on the bjdmk.com.cn AWQ article: unpack with shifts and
// masks, convert, apply the group scale and offset; here the scale and offset are applied after the
// products of each group).
//
// Nibble order. A code word holds in-features 8c .. 8c+7 in nibbles 0..7. One OR-and-mask per register
// turns the word shifted right by 4j into the bf16 pair (128 + q_j, 128 + q_{j+4}), so the operand row
// holds each word's in-features in the order 0 4 1 5 2 6 3 7. X' is permuted the same way inside every
// 16-byte chunk (8 in-features) after it lands, which leaves the products and their sum unchanged.
//
// CTA (b, c) covers weight rows [128 b, 128 b + 128) and groups [c * gp, (c + 1) * gp) (gp even). Warps:
//   0      loads: one TMA box of code words per two groups [128 rows x 32 words] (128-byte swizzle),
//          X' per group as two [nt x 64] boxes (128-byte swizzle), and the groups' steps and zero
//          points of the 128 rows (cp.async) into a ring of their own
//   1      tensor memory; per group the whole warp permutes X' in place and sums Sx_g, then one thread
//          issues the 8 MMAs (M = 128, N = nt, K = 16) into the group's accumulator
//   2-9    unpack: warps 2-5 take the first 64 in-features of every group, warps 6-9 the second; lane l
//          of warp 2 + q + 4h unpacks row 32 q + l into an operand tile (K-major, 128-byte swizzle)
//   10-13  per group: the accumulator rows of their lane quarter, times step and minus the zero-point
//          term, added to per-row registers; at the end Y (or this slice's partial sums)
// With several slices the last CTA of a row block to finish (a per-block counter it resets to zero)
// adds the slices' partial sums in slice order (deterministic). All waits are bounded; a timeout is
// recorded in the caller's status word.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace awq {
namespace dec {

constexpr int ROWS = 128;                     // weight rows per CTA (the MMA's M)
constexpr int BK = 64;                        // in-features per k-block (one 128-byte swizzle row)
constexpr int GK = 128;                       // in-features per group
constexpr int UK = 16;                        // K of one MMA
constexpr int MAX_NT = 64;                    // tokens per launch (the MMA's N, a multiple of 16)
constexpr int GROUPS_PER_BOX = 2;             // code box: 32 words = 128 bytes per row = 2 groups
constexpr int C_STAGES = 2;                   // code boxes in flight
constexpr int C_BYTES = ROWS * 128;           // 16 KB
constexpr int A_STAGES = 3;                   // unpacked operand tiles (one k-block each)
constexpr int A_BYTES = ROWS * BK * 2;        // 16 KB
constexpr int SZ_STAGES = 4;                  // steps and zero points, one group each
constexpr int SZ_BYTES = 2 * ROWS * 4;        // 1 KB
constexpr int ACC_STAGES = 4;                 // group accumulators in tensor memory
constexpr int UNPACK_WARPS = 8;
constexpr int EPI_WARP0 = 2 + UNPACK_WARPS;   // warps 10-13
constexpr int THREADS = 32 * (EPI_WARP0 + 4);  // 448
constexpr int MAX_SLICES = 16;

template <int NT>
struct Shape {
  static constexpr int X_STAGES = NT == 32 ? 2 : 4;               // X' groups in flight
  static constexpr int X_BYTES = 2 * NT * 128;                     // one group: two [NT x 64] tiles
  static constexpr int SX_STAGES = X_STAGES + ACC_STAGES;          // Sx_g ring (see the MMA warp)
  static constexpr int SMEM = C_STAGES * C_BYTES + A_STAGES * A_BYTES + X_STAGES * X_BYTES +
                              SZ_STAGES * SZ_BYTES + SX_STAGES * NT * 4 + 2 * NT * 4 + 1024;
  static constexpr int CTAS_PER_SM = NT <= 32 ? 2 : 1;
  static constexpr uint32_t TMEM_COLS = ACC_STAGES * NT <= 64 ? 64 : (ACC_STAGES * NT <= 128 ? 128 : 256);
};
static_assert(Shape<16>::SMEM <= 113 * 1024 && Shape<32>::SMEM <= 113 * 1024, "two CTAs per SM");
static_assert(Shape<64>::SMEM <= 227 * 1024, "one CTA per SM");

__host__ inline int smem_bytes(int nt) {
  return nt <= 16 ? Shape<16>::SMEM : nt <= 32 ? Shape<32>::SMEM : nt <= 48 ? Shape<48>::SMEM : Shape<64>::SMEM;
}
__host__ inline int ctas_per_sm(int nt) { return nt <= 32 ? 2 : 1; }

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
__device__ __forceinline__ bool wait_thread(uint32_t bar, uint32_t parity, const Params& p, unsigned int where) {
#pragma unroll 1
  for (int i = 0; i < 256; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
#pragma unroll 1
  while (!mbar_try_wait(bar, parity))
    if (global_timer_ns() - t0 > p.limit_ns) {
      raise_timeout(p.status, where);
      return false;
    }
  return true;
}

// Warp-uniform bounded wait: every lane polls, the warp leaves together.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const Params& p, unsigned int where) {
  // the phase has usually completed already: one poll before the timer is read
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
  if (lane == 0) t0 = global_timer_ns();
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    int give_up = 0;
    if (lane == 0 && (it & 63u) == 63u && global_timer_ns() - t0 > p.limit_ns) {
      raise_timeout(p.status, where);
      give_up = 1;
    }
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
  }
}

__device__ __forceinline__ void epilogue_sync() {  // warps 10-13 only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float ld_shared_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// (128 + q) as bf16 for the nibbles j and j + 4 of a code word shifted right by 4 j: 0x4300 | q.
__device__ __forceinline__ uint32_t nibble_pair_bf16(uint32_t w_shifted) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w_shifted));  // (a & b) | c
  return r;
}

template <int NT>
__global__ void __launch_bounds__(THREADS, Shape<NT>::CTAS_PER_SM)
    w4a16_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC, Params p) {
  using S = Shape<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * C_STAGES + 2 * A_STAGES + 3 * S::X_STAGES + 2 * SZ_STAGES +
                                        2 * ACC_STAGES];
  __shared__ uint32_t tmem_slot;
  __shared__ int failed;
  __shared__ unsigned int ticket;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = static_cast<int>(blockIdx.x) / p.slices;
  const int slice = static_cast<int>(blockIdx.x) - rb * p.slices;
  const int64_t row0 = static_cast<int64_t>(rb) * ROWS;
  const int g0 = slice * p.g_per;
  const int ng = max(0, min(p.g_per, p.num_groups - g0));  // even: num_groups and g_per are even

  const uint32_t bar0 = smem_u32(&bars[0]);
  auto cfull_bar = [&](int c) { return bar0 + 8u * c; };
  auto cempty_bar = [&](int c) { return bar0 + 8u * (C_STAGES + c); };
  auto dq_bar = [&](int a) { return bar0 + 8u * (2 * C_STAGES + a); };
  auto afree_bar = [&](int a) { return bar0 + 8u * (2 * C_STAGES + A_STAGES + a); };
  auto xfull_bar = [&](int x) { return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + x); };
  auto xempty_bar = [&](int x) { return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + S::X_STAGES + x); };
  auto szfull_bar = [&](int z) { return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + 2 * S::X_STAGES + z); };
  auto szempty_bar = [&](int z) {
    return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + 2 * S::X_STAGES + SZ_STAGES + z);
  };
  auto accfull_bar = [&](int s) {
    return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + 2 * S::X_STAGES + 2 * SZ_STAGES + s);
  };
  auto accempty_bar = [&](int s) {
    return bar0 + 8u * (2 * C_STAGES + 2 * A_STAGES + 2 * S::X_STAGES + 2 * SZ_STAGES + ACC_STAGES + s);
  };
  const uint32_t base = smem_u32(smem);
  auto c_tile = [&](int c) { return base + static_cast<uint32_t>(c) * C_BYTES; };
  auto a_tile = [&](int a) { return base + C_STAGES * C_BYTES + static_cast<uint32_t>(a) * A_BYTES; };
  auto x_tile = [&](int x, int h) {  // half h (in-features 64 h .. 64 h + 63 of the group)
    return base + C_STAGES * C_BYTES + A_STAGES * A_BYTES + static_cast<uint32_t>(x) * S::X_BYTES +
           static_cast<uint32_t>(h * NT * 128);
  };
  const uint32_t sz_base = base + C_STAGES * C_BYTES + A_STAGES * A_BYTES + S::X_STAGES * S::X_BYTES;
  auto sz_tile = [&](int z) { return sz_base + static_cast<uint32_t>(z) * SZ_BYTES; };  // [step, zero][row]
  const uint32_t sx_base = sz_base + SZ_STAGES * SZ_BYTES;
  auto sx_row = [&](int s) { return sx_base + static_cast<uint32_t>(s * NT * 4); };    // [NT] fp32
  const uint32_t px_base = sx_base + S::SX_STAGES * NT * 4;                            // [2][NT] fp32

  if (threadIdx.x == 0) {
    for (int c = 0; c < C_STAGES; ++c) {
      mbar_init(cfull_bar(c), 1);
      mbar_init(cempty_bar(c), UNPACK_WARPS);
    }
    for (int a = 0; a < A_STAGES; ++a) {
      mbar_init(dq_bar(a), UNPACK_WARPS / 2);  // the four warps of the half that writes the tile
      mbar_init(afree_bar(a), 1);
    }
    for (int x = 0; x < S::X_STAGES; ++x) {
      mbar_init(xfull_bar(x), 1);
      mbar_init(xempty_bar(x), 1);
    }
    for (int z = 0; z < SZ_STAGES; ++z) {
      mbar_init(szfull_bar(z), 32);  // the loader lanes' cp.async arrivals
      mbar_init(szempty_bar(z), 4);
    }
    for (int s = 0; s < ACC_STAGES; ++s) {
      mbar_init(accfull_bar(s), 2);  // the MMAs' commit and the MMA thread (Sx_g written)
      mbar_init(accempty_bar(s), 4);
    }
    failed = 0;
    ticket = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
  }
  // Loads of local group i: its code box when i is even (the box holds groups i and i + 1), X', and
  // the steps and zero points. Warp 0 only, all lanes; false when a wait gave up.
  auto load_codes = [&](int i) -> bool {
    const int j = i / GROUPS_PER_BOX;
    const int c = j % C_STAGES;
    const uint32_t use = static_cast<uint32_t>(j / C_STAGES);
    if (use > 0 && !wait_warp(cempty_bar(c), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(cfull_bar(c), C_BYTES);
      tma_load_2d(c_tile(c), &tmC, (g0 + i) * (GK / 8), static_cast<int32_t>(row0), cfull_bar(c));
    }
    return true;
  };
  auto load_x = [&](int i) -> bool {
    const int x = i % S::X_STAGES;
    const uint32_t use = static_cast<uint32_t>(i / S::X_STAGES);
    if (use > 0 && !wait_warp(xempty_bar(x), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(xfull_bar(x), S::X_BYTES);
      tma_load_2d(x_tile(x, 0), &tmX, (g0 + i) * GK, 0, xfull_bar(x));
      tma_load_2d(x_tile(x, 1), &tmX, (g0 + i) * GK + BK, 0, xfull_bar(x));
    }
    __syncwarp();
    return true;
  };
  auto load_sz = [&](int i) -> bool {
    const int z = i % SZ_STAGES;
    const uint32_t use = static_cast<uint32_t>(i / SZ_STAGES);
    if (use > 0 && !wait_warp(szempty_bar(z), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    const int64_t g = g0 + i;
#pragma unroll
    for (int jr = 0; jr < ROWS / 32; ++jr) {
      const int r = lane + 32 * jr;
      const int64_t o = min(row0 + r, p.O - 1);  // rows past O: any valid address (their codes are 0)
      cp_async_4(sz_tile(z) + 4u * r, p.steps + o * p.G + g);
      cp_async_4(sz_tile(z) + 4u * (ROWS + r), p.zeros + o * p.G + g);
    }
    cp_async_mbar_arrive(szfull_bar(z));
    return true;
  };
  // The first groups need no free slots: warp 0 requests them right after initialising the barriers, so
  // the first memory round trip overlaps the tensor-memory allocation and the CTA barrier.
  const int pre_c = min(ng, C_STAGES * GROUPS_PER_BOX);
  const int pre_x = min(ng, S::X_STAGES);
  const int pre_z = min(ng, SZ_STAGES);
  if (warp == 0) {
    __syncwarp();  // the barriers thread 0 initialised are visible to the whole warp
    for (int i = 0; i < pre_c; i += GROUPS_PER_BOX) load_codes(i);
    for (int i = 0; i < pre_x; ++i) load_x(i);
    for (int i = 0; i < pre_z; ++i) load_sz(i);
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------------------ loads
    for (int i = 0; i < ng; ++i) {
      bool ok = true;
      if (i >= pre_c && i % GROUPS_PER_BOX == 0) ok = load_codes(i);
      if (ok && i >= pre_x) ok = load_x(i);
      if (ok && i >= pre_z) ok = load_sz(i);
      if (!ok) {
        failed = 1;
        break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ X' and MMA
    // Per group: permute X' inside each 16-byte chunk to the unpacked operand's order 0 4 1 5 2 6 3 7
    // and sum Sx_g[m] (fp32, in a fixed order: each of the two halves in chunk and then element order,
    // then first half plus second half); then one thread issues the MMAs.
    bool ok = true;
    for (int i = 0; i < ng && ok; ++i) {
      const int x = i % S::X_STAGES;
      const int s = i % ACC_STAGES;
      if (!wait_warp(xfull_bar(x), static_cast<uint32_t>(i / S::X_STAGES) & 1u, p, kSiteDecodeFull)) {
        ok = false;
        break;
      }
#pragma unroll 1
      for (int item = lane; item < 2 * NT; item += 32) {  // (half h, token m)
        const int h = item / NT, m = item - h * NT;
        const uint32_t row = x_tile(x, h) + static_cast<uint32_t>(m) * 128u;
        float sum = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t a = row + ((static_cast<uint32_t>(c) ^ static_cast<uint32_t>(m & 7)) << 4);
          const uint4 v = ld_shared_v4(a);  // (k0 k1) (k2 k3) (k4 k5) (k6 k7)
          const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            sum = __fadd_rn(sum, __uint_as_float(e[t] << 16));
            sum = __fadd_rn(sum, __uint_as_float(e[t] & 0xFFFF0000u));
          }
          st_shared_v4(a, make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                                     __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632)));
        }
        st_shared_f32(px_base + 4u * static_cast<uint32_t>(item), sum);
      }
      fence_proxy_async_smem();  // the MMAs read the permuted X' through the async proxy
      __syncwarp();
      for (int m = lane; m < NT; m += 32)
        st_shared_f32(sx_row(i % S::SX_STAGES) + 4u * m,
                      __fadd_rn(ld_shared_f32(px_base + 4u * m), ld_shared_f32(px_base + 4u * (NT + m))));
      __syncwarp();
      if (lane == 0) {
        const int a0 = (2 * i) % A_STAGES, a1 = (2 * i + 1) % A_STAGES;
        const uint32_t acc_use = static_cast<uint32_t>(i / ACC_STAGES);
        if (!wait_thread(dq_bar(a0), static_cast<uint32_t>((2 * i) / A_STAGES) & 1u, p, kSiteDecodeDequant) ||
            !wait_thread(dq_bar(a1), static_cast<uint32_t>((2 * i + 1) / A_STAGES) & 1u, p, kSiteDecodeDequant) ||
            (acc_use > 0 && !wait_thread(accempty_bar(s), (acc_use - 1u) & 1u, p, kSiteDecodeAcc))) {
          ok = false;
        } else {
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(s * NT);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t at = a_tile(h == 0 ? a0 : a1), xt = x_tile(x, h);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk)
              umma_bf16(d, smem_desc_sw128(at + kk * UK * 2), smem_desc_sw128(xt + kk * UK * 2), p.idesc,
                        (h | kk) != 0 ? 1u : 0u);
          }
          umma_commit(afree_bar(a0));
          umma_commit(afree_bar(a1));
          umma_commit(xempty_bar(x));
          umma_commit(accfull_bar(s));
          mbar_arrive(accfull_bar(s));  // after the warp's Sx_g stores (ordered by the __syncwarp above)
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (!ok) failed = 1;
    __syncwarp();
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------------------------ unpack
    const int q = (warp - 2) & 3, h = (warp - 2) >> 2;
    const int r = 32 * q + lane;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    for (int i = 0; i < ng; ++i) {
      const int j = i / GROUPS_PER_BOX, c = j % C_STAGES;
      const int kb = 2 * i + h, a = kb % A_STAGES;
      if (!wait_warp(cfull_bar(c), static_cast<uint32_t>(j / C_STAGES) & 1u, p, kSiteDecodeFull)) {
        failed = 1;
        break;
      }
      // words 16 (i % 2) + 8 h .. + 7 of row r: 16-byte chunks 4 (i % 2) + 2 h and + 1 of its swizzled line
      const uint32_t chunk = static_cast<uint32_t>(4 * (i % GROUPS_PER_BOX) + 2 * h);
      const uint4 w0 = ld_shared_v4(c_tile(c) + static_cast<uint32_t>(r) * 128u + ((chunk ^ sw) << 4));
      const uint4 w1 = ld_shared_v4(c_tile(c) + static_cast<uint32_t>(r) * 128u + (((chunk + 1u) ^ sw) << 4));
      const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      __syncwarp();
      // the warp's last group of the box hands it back (the words are in registers)
      if (lane == 0 && (i % GROUPS_PER_BOX == GROUPS_PER_BOX - 1 || i + 1 >= ng)) mbar_arrive(cempty_bar(c));
      const uint32_t ause = static_cast<uint32_t>(kb / A_STAGES);
      if (ause > 0 && !wait_warp(afree_bar(a), (ause - 1u) & 1u, p, kSiteDecodeEmpty)) {
        failed = 1;
        break;
      }
      const uint32_t line = a_tile(a) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
      for (int t = 0; t < 8; ++t)
        st_shared_v4(line + ((static_cast<uint32_t>(t) ^ sw) << 4),
                     make_uint4(nibble_pair_bf16(w[t]), nibble_pair_bf16(w[t] >> 4), nibble_pair_bf16(w[t] >> 8),
                                nibble_pair_bf16(w[t] >> 12)));
      fence_proxy_async_smem();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_bar(a));
    }
  } else {
    // ------------------------------------------------------------------------------ group epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    const int r = 32 * q + lane;
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    float y[NT];
#pragma unroll
    for (int m = 0; m < NT; ++m) y[m] = 0.0f;
    bool have = true;
    for (int i = 0; i < ng; ++i) {
      const int z = i % SZ_STAGES, s = i % ACC_STAGES;
      if (!wait_warp(szfull_bar(z), static_cast<uint32_t>(i / SZ_STAGES) & 1u, p, kSiteDecodeFull)) {
        have = false;
        break;
      }
      const float step = ld_shared_f32(sz_tile(z) + 4u * r);
      const float c = __fadd_rn(128.0f, ld_shared_f32(sz_tile(z) + 4u * (ROWS + r)));
      __syncwarp();
      if (lane == 0) mbar_arrive(szempty_bar(z));
      if (!wait_warp(accfull_bar(s), static_cast<uint32_t>(i / ACC_STAGES) & 1u, p, kSiteDecodeAcc)) {
        have = false;
        break;
      }
      tc_fence_after();
      // 16 accumulator columns at a time: y[m] += step * (S_g[r, m] - (128 + z) * Sx_g[m])
      const uint32_t sx = sx_row(i % S::SX_STAGES);
#pragma unroll
      for (int cc = 0; cc < NT / 16; ++cc) {
        float t16[16];
        tmem_ld16(tlane + static_cast<uint32_t>(s * NT + 16 * cc), t16);
#pragma unroll
        for (int m4 = 0; m4 < 16; m4 += 4) {
          float4 xs;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(xs.x), "=f"(xs.y), "=f"(xs.z), "=f"(xs.w)
                       : "r"(sx + 4u * static_cast<uint32_t>(16 * cc + m4))
                       : "memory");
          const float xv[4] = {xs.x, xs.y, xs.z, xs.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int m = 16 * cc + m4 + k;
            y[m] = __fmaf_rn(step, __fmaf_rn(-c, xv[k], t16[m4 + k]), y[m]);
          }
        }
      }
      // The accumulator and this group's Sx_g are read: hand both back (the Sx ring is sized so that
      // its slot is rewritten only after this arrival).
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty_bar(s));
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
