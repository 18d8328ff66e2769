// kernel_loss_gemm.cuh - the reconstruction loss on the 5th-generation tensor cores.
//
// For every candidate j and every tile of 256 tokens x 256 output rows, E = X_tile * dW_tile^T is
// accumulated over K in tensor memory by a CTA pair (tcgen05.mma.cta_group::2 kind::f16, bf16 x bf16 ->
// fp32, M = 256, N = 256, K = 16 per instruction). Each CTA of the pair stages half of the X rows and
// half of the dW rows, and receives its 128 token rows of E in its own tensor memory. The epilogue
// squares and sums each row in fp32 and adds the 32 rows of each warp in fp64. E is never written to
// global memory.
//
// Persistent cooperative kernel, clusters of 2 CTAs, one CTA per SM, 14 warps per CTA. Tiles are handed
// out dynamically: the even CTA's TMA thread takes the next tile index from a global counter (the tiles
// in flight are then always a contiguous stretch of the raster, whose operands the pairs share in L2)
// and publishes it through an 8-slot ring in both CTAs' shared memory, one mbarrier per slot; -1 ends.
//   warp 0      TMA: X tile [128 x 64] and dW tile [128 x 64] per stage for this CTA, 128-byte
//               swizzle; the bytes of both CTAs are counted on the even CTA's barrier
//   warp 1      pair-wide tensor memory (512 columns = two 256-column fp32 accumulators); in the even
//               CTA one thread issues the pair MMAs and commits to barriers in both CTAs
//   warps 2-5   epilogue: one TMEM lane quarter each (warp w reads lanes 32*(w%4) .. +31)
//   warps 6-13  weight-error producers: they write dW_j (bf16, global memory) candidate by candidate,
//               all CTAs sharing each candidate's rows, and count finished rows per candidate. The
//               ALU work of the quantizer thus runs on the same SMs while the tensor cores evaluate
//               earlier candidates; the TMA warps start on candidate j once its count is complete.
// Every wait is bounded (see ptx.cuh).
#pragma once
#include <cstdint>
#include <cuda.h>

#include "kernels_simple.cuh"
#include "ptx.cuh"

namespace awq {
namespace lg {

constexpr int BM = 256;                          // tokens per pair tile (MMA M; 128 per CTA)
constexpr int BN = 256;                          // output rows per pair tile (MMA N; 128 staged per CTA)
constexpr int HALF = 128;                        // rows of each operand staged by one CTA
constexpr int BK = 64;                           // in-features per stage (one 128-byte swizzle row)
constexpr int UK = 16;                           // K of one tcgen05.mma kind::f16
constexpr int STAGES = 6;
constexpr int A_BYTES = HALF * BK * 2;           // 16 KB
constexpr int B_BYTES = HALF * BK * 2;           // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 32 KB per CTA
constexpr int NUM_ACC = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr int PROD_WARPS = 8;
constexpr int THREADS = 192 + 32 * PROD_WARPS;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + alignment slack
constexpr int PARTIALS_PER_TILE = 8;             // 2 CTAs x 4 lane quarters, 32 token rows each
constexpr int RING = 8;                          // tile-index slots; producers run <= 4 tiles ahead
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct Params {
  int n_tiles_n;      // ceil(N / BM)
  int band_begin;     // first dW band (of BN rows) this launch covers
  int n_bands;        // bands this launch covers
  int num_kb;         // K / BK
  int num_tiles;      // n_tiles_n * n_bands
  int bands_per_group;  // tile raster: this many dW bands advance together over the token blocks
  double* partials;   // [all bands][n_tiles_n][PARTIALS_PER_TILE]
  DeviceStatus* status;
  uint64_t limit_ns;
  unsigned flags;
  int tiles_o;               // bands per candidate
  int n_grid;
  ProducerArgs prod;         // weight-error production for every candidate
  int64_t items_per_cand;    // producer work items (warp x 512 in-features) per candidate
  unsigned int* produced;    // [n_grid] finished items per candidate (zeroed before launch)
  int keep_x;                // X is re-read by every band: ask L2 to keep it (evict_last)
  unsigned int* tile_counter;  // tiles handed out after each pair's first one (zeroed before launch)
};

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& band, int& nt) {
  const int per_group = p.bands_per_group * p.n_tiles_n;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int bands_in_g = min(p.bands_per_group, p.n_bands - g * p.bands_per_group);
  band = p.band_begin + g * p.bands_per_group + local % bands_in_g;
  nt = local / bands_in_g;
}

// All 32 lanes wait; the outcome is uniform across the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, DeviceStatus* st, uint64_t limit,
                                          unsigned where) {
  uint64_t t0 = 0;
  const int lane = threadIdx.x & 31;
  if (lane == 0) t0 = global_timer_ns();
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    const bool done = mbar_try_wait(bar, parity);
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

// Bounded wait until every producer warp has published candidate `cand`.
__device__ __forceinline__ bool wait_produced(const Params& p, int cand, DeviceStatus* st) {
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_u32(p.produced + cand) < static_cast<unsigned int>(p.items_per_cand)) {
    if (status_code(st) != 0u) return false;
    if (global_timer_ns() - t0 > p.limit_ns) {
      raise_timeout(st, kSiteTmaProduced);
      return false;
    }
    __nanosleep(256);
  }
  fence_proxy_async_global();
  return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    loss_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmD,
                     Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[2 * STAGES + 2 * NUM_ACC + 2 + RING];
  __shared__ uint32_t tmem_slot;
  __shared__ int tile_ring[RING];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = even CTA (issues the MMAs), 1 = odd CTA
  const uint32_t bar0 = smem_u32(&bars[0]);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + NUM_ACC + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC);
  const uint32_t never_bar = drain_bar + 8u;
  auto tile_bar = [&](int slot) { return never_bar + 8u + 8u * slot; };
  const uint32_t smem_base = smem_u32(smem);
  auto a_tile = [&](int s) { return smem_base + static_cast<uint32_t>(s) * STAGE_BYTES; };
  auto b_tile = [&](int s) { return smem_base + static_cast<uint32_t>(s) * STAGE_BYTES + A_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // the even CTA's TMA thread arms it for both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // one multicast commit per consumed stage
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 8);   // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
    for (int r = 0; r < RING; ++r) mbar_init(tile_bar(r), 1);  // the even CTA's TMA thread arrives
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(&tmem_slot), TMEM_COLS);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmD);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrive or transaction
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  DeviceStatus* st = p.status;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int n_pairs = static_cast<int>(gridDim.x >> 1);

  // Tile index of this CTA's local tile i (waits for the even CTA's TMA thread to publish it).
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

  if (warp == 0) {
    // ------------------------------------------------------------------------------ TMA
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int ready = -1;  // candidates <= ready are known to be fully produced
      // X fits L2: keep it (every band group re-reads it). Else the band group's dW rows are what the
      // tiles in flight re-read, and an X tile is used by the group's few bands right away: keep the dW,
      // let X go first.
      const uint64_t pol_x = p.keep_x ? policy_evict_last() : policy_evict_first();
      const uint64_t pol_d = p.keep_x ? policy_evict_normal() : policy_evict_last();
      for (int i = 0; ok; ++i) {
        int t;
        if (rank == 0) {
          // hand out the next tile: the pair's own first tile, then the shared counter
          t = i == 0 ? pair : n_pairs + static_cast<int>(atomicAdd(p.tile_counter, 1u));
          if (t >= p.num_tiles) t = -1;
          const int slot = i % RING;
          tile_ring[slot] = t;
          st_shared_cluster_u32(map_to_rank(smem_u32(&tile_ring[slot]), 1), static_cast<uint32_t>(t));
          mbar_arrive(tile_bar(slot));
          mbar_arrive_remote(map_to_rank(tile_bar(slot), 1));
        } else {
          t = ring_wait_thread(i, ok);
          if (!ok) break;
        }
        if (t < 0) break;
        int band, nt;
        tile_coords(t, p, band, nt);
        const int cand = band / p.tiles_o;
        if (cand > ready) {
          if (!wait_produced(p, cand, st)) {
            ok = false;
            break;
          }
          ready = cand;
        }
        const int32_t a_row = nt * BM + static_cast<int32_t>(rank) * HALF;
        const int32_t b_row = band * BN + static_cast<int32_t>(rank) * HALF;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, st, p.limit_ns, kSiteTmaEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          tma_load_2d_pair_hint(a_tile(stage), &tmX, kb * BK, a_row, fb, pol_x);
          tma_load_2d_pair_hint(b_tile(stage), &tmD, kb * BK, b_row, fb, pol_d);
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
      if (p.flags & AWQ_FLAG_INJECT_STALL) ok = mbar_wait(never_bar, 0u, st, p.limit_ns, kSiteMmaInjected);
      for (int i = 0; ok; ++i) {
        const int t = ring_wait_thread(i, ok);
        if (!ok || t < 0) break;
        const int acc = i & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(i >> 1) & 1u;
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, st, p.limit_ns, kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, st, p.limit_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = a_tile(stage), b0 = b_tile(stage);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            umma_bf16_pair(d_tmem, smem_desc_sw128(a0 + kk * UK * 2), smem_desc_sw128(b0 + kk * UK * 2), IDESC,
                           (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(accf_bar(acc), 0x3);
      }
      // Every MMA this thread issued must be complete before either CTA releases tensor memory or
      // shared memory.
      umma_commit_pair(drain_bar, 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain_bar, 0u))
        if (global_timer_ns() - t0 > p.limit_ns) {
          raise_timeout(st, kSiteDrainMma);
          break;
        }
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------------------------ producers
    // Warp v owns one segment (seg = v % segs) and every wps-th row of it, so the segment's scales are
    // loaded once per candidate; with fewer warps than segments a warp walks several whole segments.
    const int64_t v = static_cast<int64_t>(blockIdx.x) * PROD_WARPS + (warp - 6);
    const int64_t total = static_cast<int64_t>(gridDim.x) * PROD_WARPS;
    const int64_t segs = p.prod.segs;
    for (int j = 0; j < p.n_grid; ++j) {
      unsigned int done = 0;
      if (total >= segs) {
        const int64_t wps = total / segs;
        if (v < wps * segs) done = produce_rows(p.prod, v % segs, v / segs, wps, j, lane);
      } else {
        for (int64_t seg = v; seg < segs; seg += total) done += produce_rows(p.prod, seg, 0, 1, j, lane);
      }
      fence_proxy_async_global();
      __threadfence();
      __syncwarp();
      if (lane == 0 && done != 0u) atomicAdd(p.produced + j, done);
    }
  } else {
    // ------------------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    for (int i = 0;; ++i) {
      // the tile's index (all lanes wait on the ring slot; the outcome is warp-uniform)
      const int slot = i % RING;
      const uint32_t par = static_cast<uint32_t>(i / RING) & 1u;
      bool got = false;
      {
        uint64_t t0 = 0;
        if (lane == 0) t0 = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
          const bool done = mbar_try_wait_cluster(tile_bar(slot), par);
          if (__all_sync(0xffffffffu, done)) {
            got = true;
            break;
          }
          int give_up = 0;
          if (lane == 0 && (it & 63u) == 63u) {
            if (status_code(st) != 0u) give_up = 1;
            else if (global_timer_ns() - t0 > p.limit_ns) {
              raise_timeout(st, kSiteTileRing);
              give_up = 1;
            }
          }
          if (__shfl_sync(0xffffffffu, give_up, 0)) break;
        }
      }
      if (!got) break;
      const int t = *reinterpret_cast<volatile int*>(&tile_ring[slot]);
      if (t < 0) break;
      const int acc = i & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(i >> 1) & 1u;
      if (!warp_wait(accf_bar(acc), acc_phase, st, p.limit_ns, kSiteEpiAccFull)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      float sum = 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
#pragma unroll
        for (int k = 0; k < 32; ++k) sum = fmaf(v[k], v[k], sum);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(acce_bar(acc), 0));
      double ds = static_cast<double>(sum);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ds = __dadd_rn(ds, __shfl_xor_sync(0xffffffffu, ds, off));
      if (lane == 0) {
        int band, nt;
        tile_coords(t, p, band, nt);
        p.partials[(static_cast<int64_t>(band) * p.n_tiles_n + nt) * PARTIALS_PER_TILE + rank * 4 + quarter] = ds;
      }
    }
  }

  if (status_code(st) != 0u) {
    // After a timeout some copies into this CTA's shared memory may still be in flight (their
    // completion is counted on the even CTA's barrier, which may never be waited on): give them time
    // to land before the pair releases its memory.
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) __nanosleep(1000);
  }
  tc_fence_before();
  cluster_sync();  // no CTA of the pair leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace lg
}  // namespace awq
