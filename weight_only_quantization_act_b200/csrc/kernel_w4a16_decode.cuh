// kernel_w4a16_decode.cuh - the deployment GEMM of an AWQ-quantized linear for few tokens (decode, small
// batches): Y = X' deq(W)^T with M <= 64 tokens. At this size the work is reading and dequantizing the
// packed weights, so the weight rows take the MMA's M side and the k-blocks are split until every SM has
// a share:
//
//   CTA (b, c) covers weight rows [128 b, 128 b + 128) and k-blocks [c * kb_per, (c + 1) * kb_per)
//   (kb_per a multiple of 4); D[128 rows][nt tokens] accumulates in tensor memory (tcgen05.mma
//   cta_group::1, kind::f16, M = 128, N = nt = tokens rounded up to 16, K = 16) and is written to the
//   workspace as slice c of row block b; the last CTA of a row block to finish (a per-block counter,
//   which it resets to zero for the next call) adds the S slices in slice order (deterministic), converts
//   to bf16 and writes Y. With one slice the accumulator goes straight to Y.
//
// The loads are few and large, since scattered small requests are what limits this size: the code words
// of 4 k-blocks come as one TMA box [128 rows x 32 words] with 128-byte swizzle (128 contiguous bytes per
// row), with the two groups' steps and zero points of those rows (8-byte cp.async per row and array); X'
// comes per k-block [nt x 64] (128-byte swizzle) through a ring of its own.
//
// Warps: 0 loads (lane 0 the TMA boxes; all lanes the steps and zero points); 1 allocates tensor memory
// and issues the MMAs; 2-9 dequantize into a 3-deep ring of K-major swizzled operand tiles in two groups
// that take alternate k-blocks (warp 2 + q + 4g takes rows 32q..32q+31, all 64 in-features, of the
// k-blocks i with i % 2 == g, so each warp synchronises once per 64 weights of a row), computing in
// registers first and storing once the tile is free; warps 2-5 then read the accumulator (warp w may
// read tensor-memory lanes 32 (w % 4) ...). All waits are bounded; a timeout is recorded in the caller's
// status word.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "dequant_w4.cuh"
#include "ptx.cuh"

namespace awq {
namespace dec {

constexpr int ROWS = 128;                     // weight rows per CTA (the MMA's M)
constexpr int BK = 64;                        // in-features per k-block
constexpr int UK = 16;                        // K of one MMA
constexpr int MAX_NT = 64;                    // tokens per launch (the MMA's N, a multiple of 16)
constexpr int KB_PER_BOX = 4;                 // k-blocks per code box (32 words = 128 bytes per row)
constexpr int C_STAGES = 2;                   // code boxes in flight
constexpr int C_BYTES = ROWS * 128;           // 16 KB code words
constexpr int SZ_BYTES = 2 * 2 * ROWS * 4;    // 2 KB steps and zero points of the box's two groups
constexpr int C_STAGE_BYTES = C_BYTES + SZ_BYTES;
constexpr int X_STAGES = 8;                   // X' k-blocks in flight
constexpr int A_STAGES = 3;                   // dequantized operand tiles
constexpr int A_BYTES = ROWS * BK * 2;        // 16 KB dequantized weight rows
constexpr int DQ_WARPS = 8;
constexpr int THREADS = 64 + 32 * DQ_WARPS;
constexpr int TMEM_COLS = 64;                 // >= MAX_NT, a power of two >= 32
constexpr int MAX_SLICES = 16;

__host__ __device__ constexpr int x_stage_bytes(int nt) { return nt * BK * 2; }
__host__ __device__ constexpr int smem_bytes(int nt) {
  return C_STAGES * C_STAGE_BYTES + A_STAGES * A_BYTES + X_STAGES * x_stage_bytes(nt) + 1024;
}
static_assert(C_STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0 && x_stage_bytes(16) % 1024 == 0,
              "swizzled tiles stay 1024-byte aligned");
static_assert(MAX_NT * ROWS * 4 <= A_STAGES * A_BYTES, "the partial sums fit in the operand tiles' memory");

// Slices of the k-blocks per row block the workspace is sized for: enough for 512 CTAs, at most
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
  int nt;                 // MMA N: M rounded up to 16
  int num_kb;             // K / 64
  int kb_per;             // k-blocks per slice, a multiple of KB_PER_BOX
  int slices;
  int sz_pairs;           // G even and steps / zeros 8-byte aligned: one 8-byte copy per row and array
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

__device__ __forceinline__ void epilogue_sync() {  // warps 2-5 only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__global__ void __launch_bounds__(THREADS, 2)
    w4a16_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * C_STAGES + 2 * X_STAGES + 2 * A_STAGES + 1];
  __shared__ uint32_t tmem_slot;
  __shared__ int failed;
  __shared__ unsigned int ticket;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rb = static_cast<int>(blockIdx.x) / p.slices;
  const int slice = static_cast<int>(blockIdx.x) - rb * p.slices;
  const int64_t row0 = static_cast<int64_t>(rb) * ROWS;
  const int kb0 = slice * p.kb_per;
  const int nkb = max(0, min(p.kb_per, p.num_kb - kb0));
  const uint32_t xb = static_cast<uint32_t>(x_stage_bytes(p.nt));

  const uint32_t bar0 = smem_u32(&bars[0]);
  auto cfull_bar = [&](int c) { return bar0 + 8u * c; };                                   // codes landed
  auto cempty_bar = [&](int c) { return bar0 + 8u * (C_STAGES + c); };                     // codes read
  auto xfull_bar = [&](int x) { return bar0 + 8u * (2 * C_STAGES + x); };                  // X' landed
  auto xempty_bar = [&](int x) { return bar0 + 8u * (2 * C_STAGES + X_STAGES + x); };      // MMAs done with X'
  auto dq_bar = [&](int a) { return bar0 + 8u * (2 * C_STAGES + 2 * X_STAGES + a); };      // operand written
  auto afree_bar = [&](int a) { return bar0 + 8u * (2 * C_STAGES + 2 * X_STAGES + A_STAGES + a); };
  const uint32_t acc_bar = bar0 + 8u * (2 * C_STAGES + 2 * X_STAGES + 2 * A_STAGES);
  const uint32_t base = smem_u32(smem);
  auto c_tile = [&](int c) { return base + static_cast<uint32_t>(c) * C_STAGE_BYTES; };
  auto sz_tile = [&](int c) { return c_tile(c) + C_BYTES; };  // [array: step, zero][row][group 0, 1]
  auto a_tile = [&](int a) { return base + C_STAGES * C_STAGE_BYTES + static_cast<uint32_t>(a) * A_BYTES; };
  auto x_tile = [&](int x) {
    return base + C_STAGES * C_STAGE_BYTES + A_STAGES * A_BYTES + static_cast<uint32_t>(x) * xb;
  };

  if (threadIdx.x == 0) {
    for (int c = 0; c < C_STAGES; ++c) {
      mbar_init(cfull_bar(c), 1 + 32);  // the TMA arm and the 32 loader lanes' cp.async arrivals
      mbar_init(cempty_bar(c), DQ_WARPS);
    }
    for (int x = 0; x < X_STAGES; ++x) {
      mbar_init(xfull_bar(x), 1);
      mbar_init(xempty_bar(x), 1);
    }
    for (int a = 0; a < A_STAGES; ++a) {
      mbar_init(dq_bar(a), DQ_WARPS / 2);  // the four warps of the group that writes the tile
      mbar_init(afree_bar(a), 1);
    }
    mbar_init(acc_bar, 1);
    failed = 0;
    ticket = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
  }
  // Loads of k-block i: its code box when i starts one (the TMA part, then the steps and zero points),
  // and its X' tile. Warp 0 only, all lanes; false when a wait gave up.
  const bool pair_aligned = p.sz_pairs != 0;  // the box's two groups are one aligned 8-byte pair
  auto box_tma = [&](int i) -> bool {           // i a multiple of KB_PER_BOX
    const int j = i / KB_PER_BOX;
    const int c = j % C_STAGES;
    const uint32_t use = static_cast<uint32_t>(j / C_STAGES);
    if (use > 0 && !wait_warp(cempty_bar(c), (use - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(cfull_bar(c), C_BYTES);
      tma_load_2d(c_tile(c), &tmC, (kb0 + i) * (BK / 8), static_cast<int32_t>(row0), cfull_bar(c));
    }
    return true;
  };
  auto box_sz = [&](int i) {  // after box_tma(i)
    const int c = (i / KB_PER_BOX) % C_STAGES;
    const int64_t g0 = (static_cast<int64_t>(kb0 + i) * BK) >> 7;  // even: kb0 + i is a multiple of 4
#pragma unroll
    for (int jr = 0; jr < ROWS / 32; ++jr) {
      const int r = lane + 32 * jr;
      const int64_t o = min(row0 + r, p.O - 1);  // rows past O: any valid address (their codes are 0)
      const uint32_t ds = sz_tile(c) + 8u * r, dz = sz_tile(c) + 8u * (ROWS + r);
      if (pair_aligned) {
        cp_async_8(ds, p.steps + o * p.G + g0);
        cp_async_8(dz, p.zeros + o * p.G + g0);
      } else {
        cp_async_4(ds, p.steps + o * p.G + g0);
        cp_async_4(dz, p.zeros + o * p.G + g0);
        if (g0 + 1 < p.G) {
          cp_async_4(ds + 4u, p.steps + o * p.G + g0 + 1);
          cp_async_4(dz + 4u, p.zeros + o * p.G + g0 + 1);
        }
      }
    }
    cp_async_mbar_arrive(cfull_bar(c));
  };
  auto x_tma = [&](int i) -> bool {
    const int x = i % X_STAGES;
    const uint32_t xuse = static_cast<uint32_t>(i / X_STAGES);
    if (xuse > 0 && !wait_warp(xempty_bar(x), (xuse - 1u) & 1u, p, kSiteDecodeEmpty)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(xfull_bar(x), xb);
      tma_load_2d(x_tile(x), &tmX, (kb0 + i) * BK, 0, xfull_bar(x));
    }
    __syncwarp();
    return true;
  };
  // The first k-blocks need no free slots: warp 0 requests them right after initialising the barriers
  // (every TMA first, then the steps and zero points), so the first memory round trip overlaps the
  // tensor-memory allocation and the CTA barrier.
  const int pre = min(nkb, min(C_STAGES * KB_PER_BOX, X_STAGES));
  if (warp == 0) {
    __syncwarp();  // the barriers thread 0 initialised are visible to the whole warp
    for (int i = 0; i < pre; i += KB_PER_BOX) box_tma(i);
    for (int i = 0; i < pre; ++i) x_tma(i);
    for (int i = 0; i < pre; i += KB_PER_BOX) box_sz(i);
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------------------ loads
    // Box j (k-blocks 4j..4j+3 of the slice) is requested before X' of its first k-block.
    for (int i = pre; i < nkb; ++i) {
      if (i % KB_PER_BOX == 0) {
        if (!box_tma(i)) {
          failed = 1;
          break;
        }
        box_sz(i);
      }
      if (!x_tma(i)) {
        failed = 1;
        break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ MMA
    if (elect_one()) {
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int x = i % X_STAGES, a = i % A_STAGES;
        if (!wait_thread(xfull_bar(x), static_cast<uint32_t>(i / X_STAGES) & 1u, p, kSiteDecodeFull) ||
            !wait_thread(dq_bar(a), static_cast<uint32_t>(i / A_STAGES) & 1u, p, kSiteDecodeDequant)) {
          ok = false;
          failed = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk)
          umma_bf16(tmem_base, smem_desc_sw128(a_tile(a) + kk * UK * 2), smem_desc_sw128(x_tile(x) + kk * UK * 2),
                    p.idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit(xempty_bar(x));
        umma_commit(afree_bar(a));
      }
      if (ok && nkb > 0)
        umma_commit(acc_bar);
      else
        mbar_arrive(acc_bar);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------------ dequantize
    const int r = (warp & 3) * 32 + lane;  // warps 2+q and 6+q both take rows 32q ...
    const int group = (warp - 2) >> 2;     // ... of the k-blocks i with i % 2 == group, all 8 words
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    for (int i = group; i < nkb; i += 2) {
      const int j = i / KB_PER_BOX, sub = i % KB_PER_BOX;
      const int c = j % C_STAGES, a = i % A_STAGES;
      if (!wait_warp(cfull_bar(c), static_cast<uint32_t>(j / C_STAGES) & 1u, p, kSiteDecodeFull)) {
        failed = 1;
        break;
      }
      // Words 8 sub .. 8 sub + 7 of row r: 16-byte chunks 2 sub and 2 sub + 1 of the row's swizzled line.
      // "memory" keeps these loads ahead of the barrier arrive below that hands the box back.
      uint32_t w[8];
      float z, stp;
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(c_tile(c) + static_cast<uint32_t>(r) * 128u + ((static_cast<uint32_t>(2 * sub) ^ sw) << 4))
                   : "memory");
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                   : "r"(c_tile(c) + static_cast<uint32_t>(r) * 128u +
                         ((static_cast<uint32_t>(2 * sub + 1) ^ sw) << 4))
                   : "memory");
      asm volatile("ld.shared.f32 %0, [%1];"
                   : "=f"(stp)
                   : "r"(sz_tile(c) + 8u * r + 4u * (sub >> 1))
                   : "memory");
      asm volatile("ld.shared.f32 %0, [%1];"
                   : "=f"(z)
                   : "r"(sz_tile(c) + 8u * (ROWS + r) + 4u * (sub >> 1))
                   : "memory");
      uint32_t v[32];
      dequant_words<8>(w, z, stp, v);  // in registers while the operand tile may still be in use
      __syncwarp();
      // this warp's last k-block of the box (nkb is even, so each group has one in every box)
      if (lane == 0 && (sub + 2 >= KB_PER_BOX || i + 2 >= nkb)) mbar_arrive(cempty_bar(c));
      const uint32_t ause = static_cast<uint32_t>(i / A_STAGES);
      if (ause > 0 && !wait_warp(afree_bar(a), (ause - 1u) & 1u, p, kSiteDecodeEmpty)) {
        failed = 1;
        break;
      }
      store_words_sw128<8>(v, a_tile(a) + static_cast<uint32_t>(r) * 128u, r, 0);
      fence_proxy_async_smem();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_bar(a));
    }
    if (warp < 6) {
      // -------------------------------------------------------------------- accumulator out
      const bool have = wait_warp(acc_bar, 0u, p, kSiteDecodeAcc) && nkb > 0;
      if (!have && nkb > 0) failed = 1;
      tc_fence_after();
      const uint32_t tlane = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      if (p.slices == 1) {
        // One slice: the accumulator is the result; each lane writes its weight row of Y.
        const int64_t o = row0 + r;
        for (int cc = 0; cc < p.nt / 16; ++cc) {
          float v[16];
          if (have) {
            tmem_ld16(tlane + static_cast<uint32_t>(cc * 16), v);
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0.0f;
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int t = cc * 16 + k;
            if (t < p.M && o < p.O) p.Y[t * p.ldy + o] = __float2bfloat16_rn(v[k]);
          }
        }
      } else {
        // Slice `slice` of the row block's partial sums, then a ticket.
        float* mine = p.partial + (static_cast<int64_t>(rb) * p.slices + slice) * p.nt * ROWS + r;
        for (int cc = 0; cc < p.nt / 16; ++cc) {
          float v[16];
          if (have) {
            tmem_ld16(tlane + static_cast<uint32_t>(cc * 16), v);
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = 0.0f;
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) __stcg(mine + (cc * 16 + k) * ROWS, v[k]);
        }
        __threadfence();
        epilogue_sync();
        if (warp == 2 && lane == 0) {
          // Every CTA takes a ticket, even after a timeout, and the last one hands the counter back at
          // zero, so the next call needs no clearing.
          ticket = atomicAdd(p.counter + rb, 1u);
          if (ticket == static_cast<unsigned int>(p.slices - 1)) p.counter[rb] = 0u;
        }
      }
    }
  }

  __syncwarp();
  __syncthreads();
  if (p.slices > 1 && ticket == static_cast<unsigned int>(p.slices - 1)) {
    // Last slice of this row block: every other slice's sums are visible (each CTA fenced before taking
    // its ticket). The whole CTA adds them in slice order, four rows per item.
    __threadfence();
    const float* blk = p.partial + static_cast<int64_t>(rb) * p.slices * p.nt * ROWS;
    const int items = static_cast<int>(p.M) * (ROWS / 4);
    // Two items per thread per pass and eight slices per round, so up to 16 loads are in flight at once.
    for (int base_it = static_cast<int>(threadIdx.x); base_it < items; base_it += 2 * THREADS) {
      int t[2], r4[2];
      bool live[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int it = base_it + u * THREADS;
        t[u] = it / (ROWS / 4);
        r4[u] = (it - t[u] * (ROWS / 4)) * 4;
        live[u] = it < items && row0 + r4[u] < p.O;  // O % 8 == 0: four rows are all in or all out
      }
      float4 acc[2] = {make_float4(0.0f, 0.0f, 0.0f, 0.0f), make_float4(0.0f, 0.0f, 0.0f, 0.0f)};
#pragma unroll 1
      for (int c0 = 0; c0 < p.slices; c0 += 8) {
        float4 v[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            v[u][c] = live[u] && c0 + c < p.slices
                          ? __ldcg(reinterpret_cast<const float4*>(blk + (static_cast<int64_t>(c0 + c) * p.nt + t[u]) * ROWS +
                                                                   r4[u]))
                          : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (c0 + c >= p.slices) continue;
            if (c0 + c == 0) {
              acc[u] = v[u][0];  // slice order: ((s0 + s1) + s2) + ...
            } else {
              acc[u].x = __fadd_rn(acc[u].x, v[u][c].x);
              acc[u].y = __fadd_rn(acc[u].y, v[u][c].y);
              acc[u].z = __fadd_rn(acc[u].z, v[u][c].z);
              acc[u].w = __fadd_rn(acc[u].w, v[u][c].w);
            }
          }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (!live[u]) continue;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
        *reinterpret_cast<uint2*>(p.Y + t[u] * p.ldy + row0 + r4[u]) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
      }
    }
  }
  if (failed) {  // let copies still in flight land before the shared memory is given up
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace dec
}  // namespace awq
