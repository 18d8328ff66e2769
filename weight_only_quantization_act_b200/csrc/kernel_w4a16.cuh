// kernel_w4a16.cuh - the deployment GEMM of an AWQ-quantized linear: Y = X' deq(W)^T with the weights
// read as packed 4-bit codes and dequantized on the fly ("GPU 硬件级反量化算子内联融合" on the bjdmk.com.cn
// AWQ article: 4-bit weights loaded compactly, unpacked with shifts and masks, converted, multiplied by
// the group scale and offset, then fed to the tensor cores). X' is the layer input already divided by
// the AWQ scales (folded into the previous operation); deq(W)[o, k] = bf16(RN32(RN32(q - z) * step)).
//
// Persistent cooperative kernel, clusters of 2 CTAs, one CTA per SM. A tile is 512 tokens x 256 output
// rows: one dequantized weight tile (each CTA stages 128 of the 256 rows) feeds two pair MMAs, one per
// 256-token half, so every dequantized weight is used by 512 tokens. Tiles are handed out dynamically
// through an 8-slot ring (as in the loss kernel), published one tile ahead so the code loads can run
// into the next tile. Warps:
//   0      TMA: both 256-token halves of X' for this CTA's 128 rows of each (128 x 64 per half and stage,
//          128-byte swizzle; both CTAs' bytes counted on the even CTA's barrier)
//   1      pair-wide tensor memory (two 256-column fp32 accumulators, one per token half); the even CTA
//          issues the pair MMAs (tcgen05.mma.cta_group::2 kind::f16, M = 256, N = 256, K = 16)
//   2-5    epilogue: both accumulators -> bf16 -> Y through two 1 KB staging buffers per warp and TMA
//          stores of 32 rows x 16 columns (clipped at M and O), each chunk's TMEM load issued one chunk
//          ahead and the accumulators released once the last chunk is read, so the drain between tiles
//          is short
//   6      TMA of the code words [128 rows x 8 words], steps and zero points (from a group-major copy) of
//          every k-block into a ring of its own, so they are resident before the operand stage frees up
//   7-14   dequantizers, two per operand stage: warps 7+s and 11+s fill every use of stage s with 64 of the
//          CTA's 128 weight rows x 64 in-features, in the 128-byte swizzled K-major layout the MMA
//          descriptor expects, then one proxy fence and one arrive on the even CTA's full barrier. The
//          values are computed in registers as soon as the codes are in, and only stored once the stage
//          is free, so the arithmetic stays off the MMA's critical path. They issue no global loads (the
//          fence would wait for them too).
// Every wait is bounded.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "dequant_w4.cuh"
#include "kernel_loss_gemm.cuh"
#include "ptx.cuh"

namespace awq {
namespace dq {

using lg::BK;
using lg::HALF;
using lg::RING;
using lg::UK;

constexpr int TM = 512;                           // tokens per tile (two pair MMAs of M = 256)
constexpr int BMH = 256;                          // tokens per MMA
constexpr int BN = 256;                           // weight rows per tile (MMA N; 128 staged per CTA)
constexpr int STAGES = 4;
constexpr int A_BYTES = HALF * BK * 2;            // 16 KB  X' rows of one token half
constexpr int B_BYTES = HALF * BK * 2;            // 16 KB  dequantized weight rows
constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
constexpr int CSTAGES = 4;                        // code ring
constexpr int C_BYTES = HALF * (BK / 8) * 4;      // 4 KB   code words of those rows
constexpr int S_BYTES = HALF * 4;                 // 512 B  step of each row (this k-block's group)
constexpr int CSTAGE_BYTES = C_BYTES + 2 * S_BYTES;
constexpr int DQ_PER_STAGE = 2;                   // dequantizer warps per stage (each half the rows)
constexpr int DQ_WARPS = STAGES * DQ_PER_STAGE;
constexpr int THREADS = 224 + 32 * DQ_WARPS;
constexpr int Y_CHUNK = 16;                       // output columns per TMA store (32 rows x 32 bytes)
constexpr int Y_BUF_BYTES = 32 * Y_CHUNK * 2;     // 1 KB; two per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + CSTAGES * CSTAGE_BYTES + 8 * Y_BUF_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BANDS_PER_GROUP = 8;                // raster: 8 weight bands advance together over X'
constexpr uint32_t IDESC = idesc_bf16_f32(BMH, BN);
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB of dynamic shared memory");
static_assert(STAGE_BYTES % 1024 == 0 && CSTAGE_BYTES % 1024 == 0, "tiles stay 1024-byte aligned");
// A parity wait only tells the phase apart from its neighbours: a waiter must see every phase of the
// barrier it waits on. With CSTAGES a multiple of STAGES, code slot c is always read by the warps of
// operand stage c % STAGES, so they wait on each of its phases in turn (any other ratio lets a warp wait
// for fill n+2 of a slot while fill n+1, read by another stage's warps, has not landed yet, and the
// parity of fill n would pass it).
static_assert(CSTAGES % STAGES == 0, "each code slot is read by one stage's warps");

struct Params {
  __nv_bfloat16* Y;        // [M][ldy]
  int64_t M, O, K, ldy;
  int n_tiles_m;           // ceil(M / 512)
  int n_bands;             // ceil(O / 256)
  int num_kb;              // K / 64
  int num_tiles;
  unsigned int* tile_counter;  // zeroed before launch
  DeviceStatus* status;
  uint64_t limit_ns;
};

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& band, int& mt) {
  const int per_group = BANDS_PER_GROUP * p.n_tiles_m;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int bands_in_g = min(BANDS_PER_GROUP, p.n_bands - g * BANDS_PER_GROUP);
  band = g * BANDS_PER_GROUP + local % bands_in_g;
  mt = local / bands_in_g;
}

// Warp-uniform bounded wait (all lanes poll), with cluster-scope acquire when `cluster` is set.
// tcgen05.ld of 16 accumulator columns (32 lanes x 32 bit) without the wait, so the next chunk's load
// runs while the previous one is converted and stored. The registers hold the values only after
// tmem_wait_ld16 on them; passing them through that asm as read-write operands keeps every use below it.
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

__device__ __forceinline__ bool warp_wait_any(uint32_t bar, uint32_t parity, DeviceStatus* st, uint64_t limit,
                                              unsigned where, bool cluster) {
  // the phase has usually completed already: one poll before the timer is read
  if (__all_sync(0xffffffffu, cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity))) return true;
  uint64_t t0 = 0;
  const int lane = threadIdx.x & 31;
  if (lane == 0) t0 = global_timer_ns();
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    const bool done = cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    int give_up = 0;
    if (lane == 0 && (it & 63u) == 63u) {
      if (status_code(st) != 0u) give_up = 1;
      else if (global_timer_ns() - t0 > limit) {
        raise_timeout(st, where);
        give_up = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
  }
}

// Group-major copy of the per-group steps and zeros: [O][G] -> [G][O_pad] (rows past O are zeros), so that
// one TMA box brings the steps of 128 consecutive weight rows for one group.
__global__ void __launch_bounds__(256) transpose_groups_kernel(const float* __restrict__ steps,
                                                               const float* __restrict__ zeros, int64_t O,
                                                               int64_t O_pad, int64_t G, float* __restrict__ steps_t,
                                                               float* __restrict__ zeros_t) {
  const int64_t o = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t g = blockIdx.y;
  if (o >= O_pad) return;
  const bool real = o < O;
  steps_t[g * O_pad + o] = real ? steps[o * G + g] : 0.0f;
  zeros_t[g * O_pad + o] = real ? zeros[o * G + g] : 0.0f;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                      const __grid_constant__ CUtensorMap tmY, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 2 * CSTAGES + 3 + RING];
  __shared__ uint32_t tmem_slot;
  __shared__ int tile_ring[RING];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t bar0 = smem_u32(&bars[0]);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };                               // even CTA: X' + B ready
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };                   // MMAs done with stage
  auto cfull_bar = [&](int c) { return bar0 + 8u * (2 * STAGES + c); };               // codes landed
  auto cempty_bar = [&](int c) { return bar0 + 8u * (2 * STAGES + CSTAGES + c); };    // codes read
  const uint32_t accf_bar = bar0 + 8u * (2 * STAGES + 2 * CSTAGES);                   // tile accumulated
  const uint32_t acce_bar = accf_bar + 8u;                                            // accumulators read
  const uint32_t drain_bar = accf_bar + 16u;
  auto tile_bar = [&](int slot) { return drain_bar + 8u + 8u * slot; };
  const uint32_t smem_base = smem_u32(smem);
  auto a_tile = [&](int s, int h) { return smem_base + static_cast<uint32_t>(s * STAGE_BYTES + h * A_BYTES); };
  auto b_tile = [&](int s) { return smem_base + static_cast<uint32_t>(s * STAGE_BYTES + 2 * A_BYTES); };
  auto c_tile = [&](int c) { return smem_base + static_cast<uint32_t>(STAGES * STAGE_BYTES + c * CSTAGE_BYTES); };
  auto s_tile = [&](int c) { return c_tile(c) + C_BYTES; };
  auto z_tile = [&](int c) { return c_tile(c) + C_BYTES + S_BYTES; };
  auto y_buf = [&](int q, int b) {
    return smem_base + static_cast<uint32_t>(STAGES * STAGE_BYTES + CSTAGES * CSTAGE_BYTES + (2 * q + b) * Y_BUF_BYTES);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1 + 2 * DQ_PER_STAGE);  // TMA arm + the stage's dequantizer warps of both CTAs
      mbar_init(empty_bar(s), 1);
    }
    for (int c = 0; c < CSTAGES; ++c) {
      mbar_init(cfull_bar(c), 1);                    // this CTA's code loader arms it
      mbar_init(cempty_bar(c), DQ_PER_STAGE);        // the dequantizer warps that read the slot
    }
    mbar_init(accf_bar, 1);
    mbar_init(acce_bar, 8);                          // 4 epilogue warps x 2 CTAs
    mbar_init(drain_bar, 1);
    for (int r = 0; r < RING; ++r) mbar_init(tile_bar(r), 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(&tmem_slot), TMEM_COLS);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmZ);
    tma_prefetch_desc(&tmY);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  DeviceStatus* st = p.status;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int n_pairs = static_cast<int>(gridDim.x >> 1);

  auto ring_wait_thread = [&](int i, bool& ok) -> int {
    const int slot = i % RING;
    const uint32_t par = static_cast<uint32_t>(i / RING) & 1u;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_cluster(tile_bar(slot), par)) {
      if (status_code(st) != 0u || global_timer_ns() - t0 > p.limit_ns) {
        if (status_code(st) == 0u) raise_timeout(st, kSiteTileRing);
        ok = false;
        return -1;
      }
    }
    return *reinterpret_cast<volatile int*>(&tile_ring[slot]);
  };
  auto ring_wait_warp = [&](int i, bool& ok) -> int {
    const int slot = i % RING;
    const uint32_t par = static_cast<uint32_t>(i / RING) & 1u;
    if (!warp_wait_any(tile_bar(slot), par, st, p.limit_ns, kSiteTileRing, true)) {
      ok = false;
      return -1;
    }
    return *reinterpret_cast<volatile int*>(&tile_ring[slot]);
  };

  if (warp == 0) {
    // ------------------------------------------------------------------------------ TMA (X')
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint64_t pol_x = policy_evict_normal();
      // The even CTA publishes tile i + 1 when it starts tile i (tile 0 first), so the code loaders can
      // run into the next tile; -1 ends the sequence.
      auto publish = [&](int i) -> int {
        int t = i == 0 ? pair : n_pairs + static_cast<int>(atomicAdd(p.tile_counter, 1u));
        if (t >= p.num_tiles) t = -1;
        const int slot = i % RING;
        tile_ring[slot] = t;
        st_shared_cluster_u32(map_to_rank(smem_u32(&tile_ring[slot]), 1), static_cast<uint32_t>(t));
        mbar_arrive(tile_bar(slot));
        mbar_arrive_remote(map_to_rank(tile_bar(slot), 1));
        return t;
      };
      int next = rank == 0 ? publish(0) : 0;
      for (int i = 0; ok; ++i) {
        int t;
        if (rank == 0) {
          t = next;
          if (t >= 0) next = publish(i + 1);
        } else {
          t = ring_wait_thread(i, ok);
          if (!ok) break;
        }
        if (t < 0) break;
        int band, mt;
        tile_coords(t, p, band, mt);
        const int32_t a_row = mt * TM + static_cast<int32_t>(rank) * HALF;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, st, p.limit_ns, kSiteTmaEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 4 * A_BYTES);
          tma_load_2d_pair_hint(a_tile(stage, 0), &tmX, kb * BK, a_row, fb, pol_x);
          tma_load_2d_pair_hint(a_tile(stage, 1), &tmX, kb * BK, a_row + BMH, fb, pol_x);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ MMA (even CTA)
    if (rank == 0 && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int t = ring_wait_thread(i, ok);
        if (!ok || t < 0) break;
        if (i > 0 && !mbar_wait(acce_bar, static_cast<uint32_t>(i - 1) & 1u, st, p.limit_ns, kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, st, p.limit_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = b_tile(stage);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t bd = smem_desc_sw128(b0 + kk * UK * 2);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16_pair(tmem_base, smem_desc_sw128(a_tile(stage, 0) + kk * UK * 2), bd, IDESC, acc);
            umma_bf16_pair(tmem_base + BN, smem_desc_sw128(a_tile(stage, 1) + kk * UK * 2), bd, IDESC, acc);
          }
          umma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(accf_bar, 0x3);
      }
      umma_commit_pair(drain_bar, 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain_bar, 0u))
        if (global_timer_ns() - t0 > p.limit_ns) {
          raise_timeout(st, kSiteDrainMma);
          break;
        }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------------------------ TMA (codes)
    if (elect_one()) {
      bool ok = true;
      int slot = 0;
      uint32_t phase = 0;
      for (int i = 0; ok; ++i) {
        const int t = ring_wait_thread(i, ok);
        if (!ok || t < 0) break;
        int band, mt;
        tile_coords(t, p, band, mt);
        const int32_t w_row = band * BN + static_cast<int32_t>(rank) * HALF;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(cempty_bar(slot), phase ^ 1u, st, p.limit_ns, kSiteTmaProduced)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(cfull_bar(slot), CSTAGE_BYTES);
          tma_load_2d(c_tile(slot), &tmC, kb * (BK / 8), w_row, cfull_bar(slot));
          tma_load_2d(s_tile(slot), &tmS, w_row, (kb * BK) >> 7, cfull_bar(slot));
          tma_load_2d(z_tile(slot), &tmZ, w_row, (kb * BK) >> 7, cfull_bar(slot));
          if (++slot == CSTAGES) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= 7) {
    // ------------------------------------------------------------------------------ dequantizers
    // K-blocks are numbered continuously over this pair's tiles (tile i, k-block kb -> g = i * num_kb + kb);
    // operand stage g % STAGES, code slot g % CSTAGES. Warps 7+s and 11+s own stage s.
    const int s_own = (warp - 7) % STAGES;
    const int part = (warp - 7) / STAGES;  // which HALF / DQ_PER_STAGE rows of the stage this warp fills
    constexpr int RR = HALF / 32 / DQ_PER_STAGE;
    bool ok = true;
    int known_tile = -1;
    for (int64_t g = s_own, use = 0; ok; g += STAGES, ++use) {
      const int i = static_cast<int>(g / p.num_kb);
      if (i > known_tile) {
        const int t = ring_wait_warp(i, ok);
        if (!ok || t < 0) break;
        known_tile = i;
      }
      const int cs = static_cast<int>(g % CSTAGES);
      if (!warp_wait_any(cfull_bar(cs), static_cast<uint32_t>(g / CSTAGES) & 1u, st, p.limit_ns, kSiteTmaEmpty,
                         false)) {
        ok = false;
        break;
      }
      const uint32_t cbase = c_tile(cs), bbase = b_tile(s_own);
      uint32_t w[RR][8];
      float z[RR], stp[RR];
#pragma unroll
      for (int rr = 0; rr < RR; ++rr) {
        // "memory" keeps these loads ahead of the barrier arrive below that hands the slot back.
        const int r = lane + 32 * (rr + part * RR);
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[rr][0]), "=r"(w[rr][1]), "=r"(w[rr][2]), "=r"(w[rr][3])
                     : "r"(cbase + static_cast<uint32_t>(r * 32))
                     : "memory");
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[rr][4]), "=r"(w[rr][5]), "=r"(w[rr][6]), "=r"(w[rr][7])
                     : "r"(cbase + static_cast<uint32_t>(r * 32 + 16))
                     : "memory");
        asm volatile("ld.shared.f32 %0, [%1];"
                     : "=f"(stp[rr])
                     : "r"(s_tile(cs) + static_cast<uint32_t>(r * 4))
                     : "memory");
        asm volatile("ld.shared.f32 %0, [%1];"
                     : "=f"(z[rr])
                     : "r"(z_tile(cs) + static_cast<uint32_t>(r * 4))
                     : "memory");
      }
      // Dequantize into registers while the operand stage may still be in use (rows past O arrive as
      // zero codes with zero step and zero: they dequantize to 0); the code slot goes back once the
      // values are computed ...
      uint32_t v[RR][32];
#pragma unroll
      for (int rr = 0; rr < RR; ++rr) dequant_words<8>(w[rr], z[rr], stp[rr], v[rr]);
      __syncwarp();
      if (lane == 0) mbar_arrive(cempty_bar(cs));
      // ... and store once the MMAs of its previous use have completed.
      if (use > 0 && !warp_wait_any(empty_bar(s_own), static_cast<uint32_t>(use - 1) & 1u, st, p.limit_ns,
                                    kSiteMmaFull, true)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int rr = 0; rr < RR; ++rr) {
        const int r = lane + 32 * (rr + part * RR);
        store_words_sw128<8>(v[rr], bbase + static_cast<uint32_t>(r) * 128u, r, 0);
      }
      fence_proxy_async_smem();  // the tensor cores read these bytes through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(full_bar(s_own), 0));
    }
  } else {
    // ------------------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    bool ok = true;
    int stores = 0;  // TMA stores this warp has issued; buffer stores & 1
    for (int i = 0; ok; ++i) {
      const int t = ring_wait_warp(i, ok);
      if (!ok || t < 0) break;
      if (!warp_wait_any(accf_bar, static_cast<uint32_t>(i) & 1u, st, p.limit_ns, kSiteEpiAccFull, false)) break;
      tc_fence_after();
      int band, mt;
      tile_coords(t, p, band, mt);
      // 32 chunks of 16 columns: both token halves' accumulators, each chunk's TMEM load issued while the
      // previous chunk is converted and stored; the accumulators go back to the MMA warp as soon as the
      // last chunk is in registers.
      constexpr int CHUNKS = 2 * BN / Y_CHUNK;
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      auto chunk_addr = [&](int cc) {
        return tq + static_cast<uint32_t>((cc / (BN / Y_CHUNK)) * BN + (cc % (BN / Y_CHUNK)) * Y_CHUNK);
      };
      auto emit = [&](const uint32_t (&r)[16], int cc) {
        const int h = cc / (BN / Y_CHUNK), c = cc % (BN / Y_CHUNK);
        const int32_t row = mt * TM + h * BMH + static_cast<int32_t>(rank) * HALF + quarter * 32;
        uint32_t pk[Y_CHUNK / 2];
#pragma unroll
        for (int k = 0; k < Y_CHUNK / 2; ++k) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
          pk[k] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        const uint32_t buf = y_buf(quarter, stores & 1);
        if (stores >= 2) {  // the store issued two chunks ago must have read this buffer
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
        }
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(buf + 32u * lane), "r"(pk[0]), "r"(pk[1]),
                     "r"(pk[2]), "r"(pk[3])
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(buf + 32u * lane + 16u), "r"(pk[4]),
                     "r"(pk[5]), "r"(pk[6]), "r"(pk[7])
                     : "memory");
        fence_proxy_async_smem();  // the TMA reads the buffer through the async proxy
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmY, buf, band * BN + c * Y_CHUNK, row);
          bulk_commit();
        }
        ++stores;
      };
      uint32_t ra[16], rb[16];
      tmem_ld16_issue(chunk_addr(0), ra);
#pragma unroll 1
      for (int cc = 0; cc < CHUNKS; cc += 2) {
        tmem_wait_ld16(ra);
        tmem_ld16_issue(chunk_addr(cc + 1), rb);
        emit(ra, cc);
        tmem_wait_ld16(rb);
        if (cc + 2 < CHUNKS) {
          tmem_ld16_issue(chunk_addr(cc + 2), ra);
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(map_to_rank(acce_bar, 0));
        }
        emit(rb, cc + 1);
      }
    }
    if (lane == 0) bulk_wait_all();  // the staging buffers are read and Y written before the CTA ends
    __syncwarp();
  }

  if (status_code(st) != 0u) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) __nanosleep(1000);
  }
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace dq
}  // namespace awq
