// kernel_w4a16_decode.cuh - the deployment GEMM of an AWQ-quantized linear for few tokens (decode, small
// batches): Y = X' deq(W)^T with M <= 64 tokens. At this size the work is reading and dequantizing the
// packed weights, so the weight rows take the MMA's M side and the k-blocks are split until every SM has
// a share:
//
//   CTA (b, c) covers weight rows [128 b, 128 b + 128) and k-blocks [c * kb_per, (c + 1) * kb_per);
//   D[128 rows][nt tokens] accumulates in tensor memory (tcgen05.mma cta_group::1, kind::f16, M = 128,
//   N = nt = tokens rounded up to 16, K = 16) and is written to the workspace as slice c of row block b;
//   the last CTA of a row block to finish (a per-block counter) adds the S slices in slice order
//   (deterministic), converts to bf16 and writes Y.
//
// Warps: 0 loads into an 8-deep input ring (lane 0: TMA of the k-block's code words [128 rows x 8 words]
// and X' tile [nt x 64], 128-byte swizzle; all lanes: cp.async of the rows' steps and zero points straight
// from the [O][K/128] arrays), so a CTA's first 8 k-blocks are requested at once; 1 allocates tensor memory
// and issues the MMAs; 2-9 dequantize into a 3-deep ring of K-major swizzled operand tiles (warp 2 + q + 4h
// takes rows 32q..32q+31, in-features 32h..32h+31 of the k-block; then proxy fence, arrive); warps 2-5 then
// read the accumulator (warp w may read tensor-memory lanes 32 (w % 4) ...). All waits are bounded; a
// timeout is recorded in the caller's status word.
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
constexpr int IN_STAGES = 8;                  // k-blocks of inputs in flight (codes, X', steps, zeros)
constexpr int A_STAGES = 3;                   // dequantized operand tiles
constexpr int A_BYTES = ROWS * BK * 2;        // 16 KB dequantized weight rows
constexpr int C_BYTES = ROWS * (BK / 8) * 4;  // 4 KB code words
constexpr int SZ_BYTES = ROWS * 4;            // 512 B steps (as much again for the zero points)
constexpr int DQ_WARPS = 8;
constexpr int THREADS = 64 + 32 * DQ_WARPS;
constexpr int TMEM_COLS = 64;                 // >= MAX_NT, a power of two >= 32
constexpr int MAX_SLICES = 16;

// Input stage: X' tile [nt x 64] (128-byte swizzle) first, then code words, steps, zero points.
__host__ __device__ constexpr int in_stage_bytes(int nt) { return nt * BK * 2 + C_BYTES + 2 * SZ_BYTES; }
__host__ __device__ constexpr int smem_bytes(int nt) {
  return A_STAGES * A_BYTES + IN_STAGES * in_stage_bytes(nt) + 1024;
}
static_assert(in_stage_bytes(16) % 1024 == 0 && in_stage_bytes(MAX_NT) % 1024 == 0, "stages stay 1024-byte aligned");

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
  unsigned int* counter;  // [n_rb], zero at launch
  int64_t M, O, G, ldy;
  int nt;                 // MMA N: M rounded up to 16
  int num_kb;             // K / 64
  int kb_per;             // k-blocks per slice
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
  __shared__ __align__(8) uint64_t bars[2 * IN_STAGES + 2 * A_STAGES + 1];
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
  const uint32_t ib = static_cast<uint32_t>(in_stage_bytes(p.nt));
  const uint32_t x_bytes = static_cast<uint32_t>(p.nt * BK * 2);

  const uint32_t bar0 = smem_u32(&bars[0]);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };                      // inputs landed
  auto empty_bar = [&](int s) { return bar0 + 8u * (IN_STAGES + s); };       // MMAs done with X' of the stage
  auto dq_bar = [&](int a) { return bar0 + 8u * (2 * IN_STAGES + a); };      // operand tile written
  auto afree_bar = [&](int a) { return bar0 + 8u * (2 * IN_STAGES + A_STAGES + a); };  // MMAs done with it
  const uint32_t acc_bar = bar0 + 8u * (2 * IN_STAGES + 2 * A_STAGES);
  const uint32_t base = smem_u32(smem);
  auto a_tile = [&](int a) { return base + static_cast<uint32_t>(a) * A_BYTES; };
  auto x_tile = [&](int s) { return base + A_STAGES * A_BYTES + static_cast<uint32_t>(s) * ib; };
  auto c_tile = [&](int s) { return x_tile(s) + x_bytes; };
  auto s_tile = [&](int s) { return c_tile(s) + C_BYTES; };
  auto z_tile = [&](int s) { return s_tile(s) + SZ_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < IN_STAGES; ++s) {
      mbar_init(full_bar(s), 1 + 32);  // the TMA arm and the 32 loader lanes' cp.async arrivals
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < A_STAGES; ++a) {
      mbar_init(dq_bar(a), DQ_WARPS);
      mbar_init(afree_bar(a), 1);
    }
    mbar_init(acc_bar, 1);
    failed = 0;
    ticket = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------------------ loads
    for (int i = 0; i < nkb; ++i) {
      const int s = i % IN_STAGES;
      const uint32_t use = static_cast<uint32_t>(i / IN_STAGES);
      if (use > 0 && !wait_warp(empty_bar(s), (use - 1u) & 1u, p, kSiteDecodeEmpty)) {
        failed = 1;
        break;
      }
      const int kb = kb0 + i;
      if (lane == 0) {
        mbar_arrive_expect_tx(full_bar(s), C_BYTES + x_bytes);
        tma_load_2d(c_tile(s), &tmC, kb * (BK / 8), static_cast<int32_t>(row0), full_bar(s));
        tma_load_2d(x_tile(s), &tmX, kb * BK, 0, full_bar(s));
      }
      const int64_t g = (static_cast<int64_t>(kb) * BK) >> 7;
#pragma unroll
      for (int j = 0; j < ROWS / 32; ++j) {
        const int r = lane + 32 * j;
        const int64_t o = min(row0 + r, p.O - 1);  // rows past O: any valid address (their codes are 0)
        cp_async_4(s_tile(s) + 4u * r, p.steps + o * p.G + g);
        cp_async_4(z_tile(s) + 4u * r, p.zeros + o * p.G + g);
      }
      cp_async_mbar_arrive(full_bar(s));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ MMA
    if (elect_one()) {
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % IN_STAGES, a = i % A_STAGES;
        if (!wait_thread(full_bar(s), static_cast<uint32_t>(i / IN_STAGES) & 1u, p, kSiteDecodeFull) ||
            !wait_thread(dq_bar(a), static_cast<uint32_t>(i / A_STAGES) & 1u, p, kSiteDecodeDequant)) {
          ok = false;
          failed = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk)
          umma_bf16(tmem_base, smem_desc_sw128(a_tile(a) + kk * UK * 2), smem_desc_sw128(x_tile(s) + kk * UK * 2),
                    p.idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit(empty_bar(s));
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
    const int half = (warp - 2) >> 2;      // ... and split the k-block's in-features
    for (int i = 0; i < nkb; ++i) {
      const int s = i % IN_STAGES, a = i % A_STAGES;
      const uint32_t ause = static_cast<uint32_t>(i / A_STAGES);
      if (!wait_warp(full_bar(s), static_cast<uint32_t>(i / IN_STAGES) & 1u, p, kSiteDecodeFull)) {
        failed = 1;
        break;
      }
      uint32_t w[4];
      float z, stp;
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(c_tile(s) + static_cast<uint32_t>(r * 32 + half * 16)));
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(stp) : "r"(s_tile(s) + 4u * r));
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(z) : "r"(z_tile(s) + 4u * r));
      uint32_t v[16];
      dequant_words<4>(w, z, stp, v);  // in registers while the operand tile may still be in use
      if (ause > 0 && !wait_warp(afree_bar(a), (ause - 1u) & 1u, p, kSiteDecodeEmpty)) {
        failed = 1;
        break;
      }
      store_words_sw128<4>(v, a_tile(a) + static_cast<uint32_t>(r) * 128u, r, 4 * half);
      fence_proxy_async_smem();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_bar(a));
    }
    if (warp < 6) {
      // -------------------------------------------------------------------- accumulator -> workspace
      const bool have = wait_warp(acc_bar, 0u, p, kSiteDecodeAcc) && nkb > 0;
      if (!have && nkb > 0) failed = 1;
      tc_fence_after();
      float* mine = p.partial + (static_cast<int64_t>(rb) * p.slices + slice) * p.nt * ROWS + r;
      for (int c = 0; c < p.nt / 16; ++c) {
        float v[16];
        if (have) {
          tmem_ld16(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + static_cast<uint32_t>(c * 16), v);
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = 0.0f;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) __stcg(mine + (c * 16 + k) * ROWS, v[k]);
      }
      __threadfence();
      epilogue_sync();
      if (warp == 2 && lane == 0) ticket = atomicAdd(p.counter + rb, 1u);
    }
  }

  __syncwarp();
  __syncthreads();
  if (ticket == static_cast<unsigned int>(p.slices - 1)) {
    // Last slice of this row block: every other slice's sums are visible (each CTA fenced before taking
    // its ticket). The whole CTA adds them in slice order, four rows per item, all slices' loads in flight.
    __threadfence();
    const float* blk = p.partial + static_cast<int64_t>(rb) * p.slices * p.nt * ROWS;
    const int items = static_cast<int>(p.M) * (ROWS / 4);
    for (int it = threadIdx.x; it < items; it += THREADS) {
      const int t = it / (ROWS / 4);
      const int r4 = (it - t * (ROWS / 4)) * 4;
      const int64_t o = row0 + r4;
      if (o >= p.O) continue;  // O % 8 == 0: four rows are all in or all out
      float4 v[MAX_SLICES];
#pragma unroll
      for (int c = 0; c < MAX_SLICES; ++c)
        v[c] = c < p.slices ? __ldcg(reinterpret_cast<const float4*>(blk + (static_cast<int64_t>(c) * p.nt + t) * ROWS + r4))
                            : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float4 acc = v[0];
#pragma unroll
      for (int c = 1; c < MAX_SLICES; ++c)
        if (c < p.slices) {
          acc.x = __fadd_rn(acc.x, v[c].x);
          acc.y = __fadd_rn(acc.y, v[c].y);
          acc.z = __fadd_rn(acc.z, v[c].z);
          acc.w = __fadd_rn(acc.w, v[c].w);
        }
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      *reinterpret_cast<uint2*>(p.Y + t * p.ldy + o) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
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
