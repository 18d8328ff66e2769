// kernels_simple.cuh - the HBM- and ALU-bound kernels of the AWQ search: activation statistic, scale
// table, weight-error producer, loss/argmin finalisation and the INT4 pack.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "numerics.cuh"
#include "ptx.cuh"

namespace awq {

// ===================================================================================================
// (1) activation statistic: act_mean[k] = RN32(RN64(S_k / N)), S_k = sum_i |X[i,k]| in fp64 in a fixed
// order (256-row chunks; rows in increasing order inside a chunk; chunk totals in chunk order).
// ===================================================================================================
constexpr int kMaxGrid = 64;  // largest n_grid (AWQ_MAX_N_GRID)
constexpr int kActChunk = 256;       // rows per chunk of the fixed-order sum
constexpr int kActCols = 8;          // adjacent columns per thread: one 16-byte load per row
constexpr int kActThreads = 64;
constexpr int kActColsPerBlock = kActThreads * kActCols;  // 512 columns per work item
constexpr int kActRowsAhead = 4;     // rows per block of loads (two blocks in flight per thread)
constexpr int kActCtasPerSm = 16;    // resident CTAs per SM the host sizes the grid for

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int Pending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(Pending) : "memory");
}

// 16 bytes that are read once: not kept in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// The magnitude of a bf16 as a double scaled by 2^-896: the bf16's 15 magnitude bits moved to the top of
// the double (its 8-bit exponent field becomes the low bits of the double's 11-bit one, its 7 mantissa
// bits the leading mantissa bits), i.e. |x| * 2^(127 - 1023) exactly, zero and subnormal bf16 values
// included (they become zero and subnormal doubles). This replaces a conversion instruction per element
// by an AND and a multiply on the integer and FMA pipes. Finite inputs only (the interface's contract).
//
// Sums of these are exactly 2^-896 times the fp64 sums of the unscaled values in the same order: the
// addends are non-negative, so a running sum only grows; while it is below 2^-1022 (scaled) every sum of
// bf16 magnitudes is exact in both scalings (multiples of 2^-133 with few significant bits), and from
// there on every result is a normal double in both, where rounding commutes with the power-of-two scale.
__device__ __forceinline__ double scaled_abs_lo(uint32_t w) { return __hiloint2double((w & 0x7FFFu) * 8192u, 0); }
__device__ __forceinline__ double scaled_abs_hi(uint32_t w) {
  return __hiloint2double(__umulhi(w & 0x7FFF0000u, 1u << 29), 0);
}
constexpr double kActUnscale = 0x1p896;

__device__ __forceinline__ void add_row8(double (&acc)[kActCols], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = __dadd_rn(acc[2 * i], scaled_abs_lo(w[i]));
    acc[2 * i + 1] = __dadd_rn(acc[2 * i + 1], scaled_abs_hi(w[i]));
  }
}

// Work item (chunk ch, column block cb) = rows [256 ch, 256 ch + 256) x columns [512 cb, 512 cb + 512);
// items are numbered chunk-major and CTA b takes items b, b + gridDim.x, ... Thread t sums its 8 adjacent
// columns down the chunk, one row at a time in increasing order (fp64, scaled by 2^-896), from 16-byte
// loads in blocks of 4 rows, the next block's loads issued before the current block's additions, and
// writes the 8 scaled chunk sums to part[ch][k]. K is even, so a ragged last column block ends on a whole
// pair; its thread reads pairs with 4-byte loads.
__global__ void __launch_bounds__(kActThreads) act_chunk_sums_kernel(const uint16_t* __restrict__ X,
                                                                     int64_t N, int64_t K, int64_t ldx,
                                                                     double* __restrict__ part) {
  constexpr int B = kActRowsAhead;
  const int64_t nx = (K + kActColsPerBlock - 1) / kActColsPerBlock;
  const int64_t items = nx * ((N + kActChunk - 1) / kActChunk);
#pragma unroll 1
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t ch = it / nx;
    const int64_t c = (it - ch * nx) * kActColsPerBlock + static_cast<int64_t>(threadIdx.x) * kActCols;
    if (c >= K) continue;
    const int64_t r0 = ch * kActChunk;
    const int nr = static_cast<int>(min(static_cast<int64_t>(kActChunk), N - r0));
    const uint16_t* p = X + r0 * ldx + c;
    double acc[kActCols];
#pragma unroll
    for (int j = 0; j < kActCols; ++j) acc[j] = 0.0;
    if (c + kActCols <= K) {
      const int nb = nr / B;  // whole blocks; the last nr % B rows follow one at a time
      uint4 va[B], vb[B];
      if (nb > 0) {
#pragma unroll
        for (int u = 0; u < B; ++u) va[u] = ld_stream16(p + u * ldx);
      }
#pragma unroll 1
      for (int b = 0; b < nb; b += 2) {
        if (b + 1 < nb) {
#pragma unroll
          for (int u = 0; u < B; ++u) vb[u] = ld_stream16(p + ((b + 1) * B + u) * ldx);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) add_row8(acc, va[u]);
        if (b + 2 < nb) {
#pragma unroll
          for (int u = 0; u < B; ++u) va[u] = ld_stream16(p + ((b + 2) * B + u) * ldx);
        }
        if (b + 1 < nb) {
#pragma unroll
          for (int u = 0; u < B; ++u) add_row8(acc, vb[u]);
        }
      }
#pragma unroll 1
      for (int r = nb * B; r < nr; ++r) add_row8(acc, ld_stream16(p + r * ldx));
      double2* out = reinterpret_cast<double2*>(part + ch * K + c);  // K even, c % 8 == 0: 16-byte aligned
#pragma unroll
      for (int j = 0; j < kActCols / 2; ++j) out[j] = make_double2(acc[2 * j], acc[2 * j + 1]);
    } else {
      const int pairs = static_cast<int>((K - c) / 2);  // 1 to 3
#pragma unroll 1
      for (int r = 0; r < nr; ++r) {
        const uint32_t* q = reinterpret_cast<const uint32_t*>(p + r * ldx);
#pragma unroll
        for (int i = 0; i < kActCols / 2; ++i)
          if (i < pairs) {
            const uint32_t w = __ldg(q + i);
            acc[2 * i] = __dadd_rn(acc[2 * i], scaled_abs_lo(w));
            acc[2 * i + 1] = __dadd_rn(acc[2 * i + 1], scaled_abs_hi(w));
          }
      }
#pragma unroll
      for (int i = 0; i < kActCols / 2; ++i)
        if (i < pairs) {
          part[ch * K + c + 2 * i] = acc[2 * i];
          part[ch * K + c + 2 * i + 1] = acc[2 * i + 1];
        }
    }
  }
}

// The same sums for layers with few work items (fewer than four of the 512-column items per SM, e.g. a
// 4096 x 4096 X): 2 adjacent columns per thread (one 4-byte load per row), 128 threads (256 columns) per
// item and 16-row blocks, so that a thread has up to 32 rows in flight and a chunk costs 8 memory round
// trips instead of 32. Same order of additions, same results.
constexpr int kActNarrowThreads = 128;
constexpr int kActNarrowColsPerBlock = 2 * kActNarrowThreads;  // 256 columns per work item
constexpr int kActNarrowRows = 16;
constexpr int kActNarrowCtasPerSm = 8;

__device__ __forceinline__ uint32_t ld_stream4(const void* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kActNarrowThreads) act_chunk_sums_narrow_kernel(const uint16_t* __restrict__ X,
                                                                                  int64_t N, int64_t K,
                                                                                  int64_t ldx,
                                                                                  double* __restrict__ part) {
  constexpr int B = kActNarrowRows;
  const int64_t nx = (K + kActNarrowColsPerBlock - 1) / kActNarrowColsPerBlock;
  const int64_t items = nx * ((N + kActChunk - 1) / kActChunk);
#pragma unroll 1
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t ch = it / nx;
    const int64_t c = (it - ch * nx) * kActNarrowColsPerBlock + 2 * static_cast<int64_t>(threadIdx.x);
    if (c >= K) continue;  // K even: columns c and c + 1 are both in
    const int64_t r0 = ch * kActChunk;
    const int nr = static_cast<int>(min(static_cast<int64_t>(kActChunk), N - r0));
    const uint16_t* p = X + r0 * ldx + c;
    double lo = 0.0, hi = 0.0;
    const int nb = nr / B;
    uint32_t va[B], vb[B];
    if (nb > 0) {
#pragma unroll
      for (int u = 0; u < B; ++u) va[u] = ld_stream4(p + u * ldx);
    }
#pragma unroll 1
    for (int b = 0; b < nb; b += 2) {
      if (b + 1 < nb) {
#pragma unroll
        for (int u = 0; u < B; ++u) vb[u] = ld_stream4(p + ((b + 1) * B + u) * ldx);
      }
#pragma unroll
      for (int u = 0; u < B; ++u) {
        lo = __dadd_rn(lo, scaled_abs_lo(va[u]));
        hi = __dadd_rn(hi, scaled_abs_hi(va[u]));
      }
      if (b + 2 < nb) {
#pragma unroll
        for (int u = 0; u < B; ++u) va[u] = ld_stream4(p + ((b + 2) * B + u) * ldx);
      }
      if (b + 1 < nb) {
#pragma unroll
        for (int u = 0; u < B; ++u) {
          lo = __dadd_rn(lo, scaled_abs_lo(vb[u]));
          hi = __dadd_rn(hi, scaled_abs_hi(vb[u]));
        }
      }
    }
#pragma unroll 1
    for (int r = nb * B; r < nr; ++r) {
      const uint32_t w = ld_stream4(p + r * ldx);
      lo = __dadd_rn(lo, scaled_abs_lo(w));
      hi = __dadd_rn(hi, scaled_abs_hi(w));
    }
    *reinterpret_cast<double2*>(part + ch * K + c) = make_double2(lo, hi);  // K, c even: 16-byte aligned
  }
}

// grid ceil(K / 256) of 256 threads: the scaled chunk totals in chunk order (exactly 2^-896 times the
// unscaled fp64 sum, by the argument above), the exact power-of-two unscale, then the mean. Eight
// chunks' loads are in flight per thread; the additions stay in chunk order.
constexpr int kActFinalizeThreads = 256;
__global__ void __launch_bounds__(kActFinalizeThreads) act_finalize_kernel(const double* __restrict__ part, int64_t N,
                                                                           int64_t K, int n_chunks,
                                                                           float* __restrict__ act_mean) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * kActFinalizeThreads + threadIdx.x;
  if (k >= K) return;
  double S = 0.0;
  for (int c = 0; c < n_chunks; c += 8) {
    double v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = c + u < n_chunks ? __ldcg(part + static_cast<int64_t>(c + u) * K + k) : 0.0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c + u < n_chunks) S = __dadd_rn(S, v[u]);
  }
  act_mean[k] = __double2float_rn(__ddiv_rn(__dmul_rn(S, kActUnscale), static_cast<double>(N)));
}

// ===================================================================================================
// (2) scale table: t = CR32(act^r) clamped at 1e-4, then t / sqrt(max t * min t) per row j.
// ===================================================================================================
constexpr int kScaleThreads = 256;

__device__ __forceinline__ void block_max_min(float& mx, float& mn, float* red /* [2 * 32] */) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    red[w] = mx;
    red[32 + w] = mn;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    mx = l < nw ? red[l] : 0.0f;
    mn = l < nw ? red[32 + l] : __int_as_float(0x7f800000);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
  }
}

// Candidate-scale rules (the `mode` of the scale kernels).
enum ScaleMode : int {
  kScalesP4 = 0,           // clamp(act^(j/n), 1e-4) / sqrt(max * min)
  kScalesWeightAware = 1,  // clamp(act^p / (wmean^(1-p) + 1e-6), 1e-4) / sqrt(max * min), p = j/(n-1)
  kScalesRms = 2,          // clamp(max(act, 1e-5)^a / sqrt(mean(s^2)), 1e-4), a = j/(n-1)
};

__device__ __forceinline__ float closed_grid(int j, int n_grid) {
  return n_grid == 1 ? 0.0f : __fdiv_rn(static_cast<float>(j), static_cast<float>(n_grid - 1));
}

// grid (ceil(K / 256), n_grid). Modes P4 / weight-aware: t (clamped) to the table, per-block max/min to
// part (float2). RMS mode: t (unclamped) to the table, the fp64 sum of RN32(t^2) over the block's 256
// columns in column order to part (as a double).
__global__ void __launch_bounds__(kScaleThreads) scale_pow_kernel(const float* __restrict__ act,
                                                                  const float* __restrict__ wmean, int64_t K,
                                                                  int n_grid, int mode, int force_slow,
                                                                  float* __restrict__ table,
                                                                  float2* __restrict__ part) {
  __shared__ float red[64];
  __shared__ float sq[kScaleThreads];
  const int j = blockIdx.y;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * kScaleThreads + threadIdx.x;
  const bool slow = force_slow != 0;
  float t = 0.0f;
  if (k < K) {
    if (mode == kScalesP4) {
      const float r = __fdiv_rn(static_cast<float>(j), static_cast<float>(n_grid));
      t = fmaxf(pow_f32_cr(act[k], r, slow), AWQ_SCALE_FLOOR);
    } else if (mode == kScalesWeightAware) {
      const float p = closed_grid(j, n_grid);
      const float tp = pow_f32_cr_full(act[k], p, slow);
      const float u = pow_f32_cr_full(wmean[k], __fsub_rn(1.0f, p), slow);
      t = fmaxf(__fdiv_rn(tp, __fadd_rn(u, AWQ_WEIGHT_EPS)), AWQ_SCALE_FLOOR);
    } else {
      t = pow_f32_cr_full(fmaxf(act[k], AWQ_RMS_ACT_FLOOR), closed_grid(j, n_grid), slow);
    }
    table[static_cast<int64_t>(j) * K + k] = t;
  }
  if (mode == kScalesRms) {
    sq[threadIdx.x] = __fmul_rn(t, t);  // columns past K contribute +0
    __syncthreads();
    if (threadIdx.x == 0) {
      double acc = 0.0;
      for (int i = 0; i < kScaleThreads; ++i) acc = __dadd_rn(acc, static_cast<double>(sq[i]));
      reinterpret_cast<double*>(part)[static_cast<int64_t>(j) * gridDim.x + blockIdx.x] = acc;
    }
    return;
  }
  float mx = k < K ? t : 0.0f, mn = k < K ? t : __int_as_float(0x7f800000);
  block_max_min(mx, mn, red);
  if (threadIdx.x == 0) part[static_cast<int64_t>(j) * gridDim.x + blockIdx.x] = make_float2(mx, mn);
}

// grid (ceil(K / 256), n_grid): every block reduces the row's partials (cheap, <= a few hundred entries)
// and normalises its 256 columns in place. Optionally also writes RN32(1/s) for the producer.
__global__ void __launch_bounds__(kScaleThreads) scale_normalize_kernel(float* __restrict__ table,
                                                                        float* __restrict__ rtable,
                                                                        const float2* __restrict__ part,
                                                                        int64_t K, int nblk, int mode) {
  __shared__ float red[64];
  __shared__ float d_sh;
  const int j = blockIdx.y;
  if (mode == kScalesRms) {
    if (threadIdx.x == 0) {
      double S = 0.0;  // chunk totals in chunk order
      const double* ps = reinterpret_cast<const double*>(part) + static_cast<int64_t>(j) * nblk;
      for (int b = 0; b < nblk; ++b) S = __dadd_rn(S, ps[b]);
      d_sh = __fsqrt_rn(__double2float_rn(__ddiv_rn(S, static_cast<double>(K))));
    }
  } else {
    float mx = 0.0f, mn = __int_as_float(0x7f800000);
    for (int b = threadIdx.x; b < nblk; b += blockDim.x) {
      const float2 v = part[static_cast<int64_t>(j) * nblk + b];
      mx = fmaxf(mx, v.x);
      mn = fminf(mn, v.y);
    }
    block_max_min(mx, mn, red);
    if (threadIdx.x == 0) d_sh = __fsqrt_rn(__fmul_rn(mx, mn));
  }
  __syncthreads();
  const float d = d_sh;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * kScaleThreads + threadIdx.x;
  if (k < K) {
    const int64_t idx = static_cast<int64_t>(j) * K + k;
    float s = __fdiv_rn(table[idx], d);
    if (mode == kScalesRms) s = fmaxf(s, AWQ_SCALE_FLOOR);
    table[idx] = s;
    if (rtable != nullptr) rtable[idx] = __frcp_rn(s);
  }
}

// ===================================================================================================
// (3) weight-error producer: dW_j[o, k] = bf16(RN32(w - w_hat_j)), written as the B operand of the loss
// GEMM (row j * O_pad + o, K contiguous); rows o >= O are written as zeros. A work item is 512
// consecutive in-features (a segment) of one row, done by one warp: each lane owns 16 in-features
// (8 lanes per group of 128). The producer warps of the loss-GEMM kernel call produce_rows.
// w_hat = deq * RN32(1/s) by default (within one fp32 rounding of deq / s; it only feeds the loss);
// with AWQ_FLAG_EXACT_DIVISION it is the IEEE quotient RN32(deq / s) of the method's unscale step.
// ===================================================================================================
constexpr int kProdCols = 16;
constexpr int kProdWarpCols = 32 * kProdCols;  // 512

struct ProducerArgs {
  const uint16_t* W;
  int64_t O, O_pad, K, ldw, segs;  // segs = ceil(K / 512) items per row
  const float* table;              // [n_grid][K] scales
  const float* rtable;             // [n_grid][K] RN32(1 / scale)
  __nv_bfloat16* dW;               // [n_grid * O_pad][K]
  int exact;                       // AWQ_FLAG_EXACT_DIVISION
  int keep_w;                      // W is re-read once per candidate: ask L2 to keep it (evict_last)
  const float* rowstep;            // INT8 per-channel quantizer: [n_grid][O_pad] steps, else null
};

// w_hat from the dequantized value: deq * RN32(1/s), or the IEEE quotient deq / s when exact.
__device__ __forceinline__ float unscale(float deq, float s, float rs, bool exact) {
  return exact ? __fdiv_rn(deq, s) : __fmul_rn(deq, rs);
}

// Weight errors of one row of one 512-in-feature segment for candidate j, from the row's raw bf16 words.
__device__ __forceinline__ void produce_row(const ProducerArgs& a, const uint4 (&u)[2], const float (&s)[kProdCols],
                                            const float (&rs)[kProdCols], bool real_row, float row_step,
                                            uint32_t (&outw)[8]) {
  if (!real_row) {  // padding rows (o >= O) are zeros; warp-uniform
#pragma unroll
    for (int i = 0; i < 8; ++i) outw[i] = 0u;
    return;
  }
  const uint32_t raw[8] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w};
  float w[kProdCols], wp[kProdCols];
  float mx = -__int_as_float(0x7f800000), mn = __int_as_float(0x7f800000);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w[2 * i] = bf16_lo(raw[i]);
    w[2 * i + 1] = bf16_hi(raw[i]);
    fx2_split(fx2_mul(fx2(w[2 * i], w[2 * i + 1]), fx2(s[2 * i], s[2 * i + 1])), wp[2 * i], wp[2 * i + 1]);
    mx = max3f(mx, wp[2 * i], wp[2 * i + 1]);
    mn = min3f(mn, wp[2 * i], wp[2 * i + 1]);
  }
  if (a.rowstep != nullptr) {  // INT8 per-channel: the row's step comes from the pre-pass
    GroupParams g;
    g.step = row_step;
    g.zero = 0.0f;
    g.rstep = __frcp_rn(row_step);
#pragma unroll
    for (int i = 0; i < kProdCols; i += 2) {
      const float q0 = code_of_int8(wp[i], g, a.exact != 0), q1 = code_of_int8(wp[i + 1], g, a.exact != 0);
      const float h0 = unscale(__fmul_rn(q0, g.step), s[i], rs[i], a.exact != 0);
      const float h1 = unscale(__fmul_rn(q1, g.step), s[i + 1], rs[i + 1], a.exact != 0);
      const __nv_bfloat162 pr = __floats2bfloat162_rn(__fsub_rn(w[i], h0), __fsub_rn(w[i + 1], h1));
      outw[i / 2] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    return;
  }
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
  }
  const GroupParams g = group_params(mx, mn);
  float C = 0.0f;
  if (a.exact == 0 && fast_group(g, mx, mn, C)) {
    // Fast path (see fast_group): r = rint(w' / step) from t = RN(RN(w' * rstep) + C), deq = RN(r * step),
    // w_hat = RN(deq * RN(1/s)), dW = bf16(RN(w - w_hat)), two elements per paired instruction.
    const uint64_t rs2 = fx2(g.rstep, g.rstep), C2 = fx2(C, C), st2 = fx2(g.step, g.step);
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < kProdCols; i += 2) {
      const uint64_t qa = fx2_mul(fx2(wp[i], wp[i + 1]), rs2);
      const uint64_t r = fx2_sub(fx2_add(qa, C2), C2);
      float d0, d1;
      fx2_split(fx2_sub(qa, r), d0, d1);
      dmax = max3f(dmax, fabsf(d0), fabsf(d1));
      const uint64_t w_hat = fx2_mul(fx2_mul(r, st2), fx2(rs[i], rs[i + 1]));
      float e0, e1;
      fx2_split(fx2_sub(fx2(w[i], w[i + 1]), w_hat), e0, e1);
      const __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
      outw[i / 2] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    if (dmax < kTieMargin) return;  // else: a quotient near a half-integer, redo the lane exactly
  }
#pragma unroll
  for (int i = 0; i < kProdCols; i += 2) {
    const float q0 = code_of(wp[i], g, a.exact != 0), q1 = code_of(wp[i + 1], g, a.exact != 0);
    const float h0 = unscale(dequant(q0, g), s[i], rs[i], a.exact != 0);
    const float h1 = unscale(dequant(q1, g), s[i + 1], rs[i + 1], a.exact != 0);
    const __nv_bfloat162 pr = __floats2bfloat162_rn(__fsub_rn(w[i], h0), __fsub_rn(w[i + 1], h1));
    outw[i / 2] = *reinterpret_cast<const uint32_t*>(&pr);
  }
}

// Rows o_first, o_first + o_step, ... < O_pad of segment `seg` for candidate j. The segment's scales
// stay in registers; the next row's weights are loaded while the current row is computed. Returns the
// number of (row, segment) items written.
__device__ __forceinline__ unsigned int produce_rows(const ProducerArgs& a, int64_t seg, int64_t o_first,
                                                     int64_t o_step, int j, int lane) {
  const int64_t k0 = seg * kProdWarpCols + static_cast<int64_t>(lane) * kProdCols;
  const bool active = k0 < a.K;  // K % 128 == 0: 8-lane groups are all active or all idle
  float s[kProdCols], rs[kProdCols];
  if (active) {
    const float4* ps = reinterpret_cast<const float4*>(a.table + static_cast<int64_t>(j) * a.K + k0);
    const float4* pr = reinterpret_cast<const float4*>(a.rtable + static_cast<int64_t>(j) * a.K + k0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = __ldg(ps + i), y = __ldg(pr + i);
      s[4 * i] = x.x; s[4 * i + 1] = x.y; s[4 * i + 2] = x.z; s[4 * i + 3] = x.w;
      rs[4 * i] = y.x; rs[4 * i + 1] = y.y; rs[4 * i + 2] = y.z; rs[4 * i + 3] = y.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kProdCols; ++i) { s[i] = 1.0f; rs[i] = 1.0f; }
  }
  unsigned int count = 0;
  const uint64_t pol = a.keep_w ? policy_evict_last() : policy_evict_normal();
  uint4 nxt[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  if (o_first < a.O && active) {
    const uint4* src = reinterpret_cast<const uint4*>(a.W + o_first * a.ldw + k0);
    nxt[0] = ldg_v4_policy(src, pol);
    nxt[1] = ldg_v4_policy(src + 1, pol);
  }
  for (int64_t o = o_first; o < a.O_pad; o += o_step) {
    const uint4 cur[2] = {nxt[0], nxt[1]};
    const int64_t on = o + o_step;
    if (on < a.O && active) {
      const uint4* src = reinterpret_cast<const uint4*>(a.W + on * a.ldw + k0);
      nxt[0] = ldg_v4_policy(src, pol);
      nxt[1] = ldg_v4_policy(src + 1, pol);
    }
    uint32_t outw[8];
    const float row_step = a.rowstep != nullptr ? __ldg(a.rowstep + static_cast<int64_t>(j) * a.O_pad + o) : 0.0f;
    produce_row(a, cur, s, rs, o < a.O, row_step, outw);
    if (active) {
      uint4* dst = reinterpret_cast<uint4*>(a.dW + (static_cast<int64_t>(j) * a.O_pad + o) * a.K + k0);
      dst[0] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
      dst[1] = make_uint4(outw[4], outw[5], outw[6], outw[7]);
    }
    ++count;
  }
  return count;
}

// ===================================================================================================
// (4)-(5) finalisation: loss_j = (sum of the tile partials in a fixed order) / (N * O); best_j is the
// first index of the minimum; scales = row best_j of the table. Single block of 1024 threads.
// ===================================================================================================
// grid n_grid blocks of 256: block j sums candidate j's tile partials in a fixed order (thread t takes
// entries t, t + 256, ... in order; then a fixed tree), so the result does not depend on scheduling. The
// last block to finish (counter in the zeroed status block) takes the first minimum and copies the
// scales of the best ratio.
constexpr int kFinThreads = 256;

__global__ void __launch_bounds__(kFinThreads) finalize_kernel(const double* __restrict__ partials,
                                                               int64_t per_cand, int n_grid, double denom,
                                                               const float* __restrict__ table, int64_t K,
                                                               double* __restrict__ losses, int* __restrict__ best_j,
                                                               float* __restrict__ scales, const DeviceStatus* st,
                                                               unsigned int* done_blocks) {
  __shared__ double red[kFinThreads];
  __shared__ int last_sh;
  __shared__ int best_sh;
  const int j = blockIdx.x;
  const bool failed = status_code(st) != 0u;
  double acc = 0.0;
  const double* p = partials + static_cast<int64_t>(j) * per_cand;
  for (int64_t i = threadIdx.x; i < per_cand; i += kFinThreads) acc = __dadd_rn(acc, p[i]);
  red[threadIdx.x] = acc;
  __syncthreads();
#pragma unroll
  for (int w = kFinThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = __dadd_rn(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    losses[j] = failed ? __longlong_as_double(0x7ff8000000000000ll) : __ddiv_rn(red[0], denom);
    __threadfence();
    last_sh = atomicAdd(done_blocks, 1u) == static_cast<unsigned int>(n_grid - 1);
  }
  __syncthreads();
  if (!last_sh) return;
  __threadfence();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    double v = __longlong_as_double(0x7ff0000000000000ll);
    int idx = 0x7fffffff;
    for (int c = lane; c < n_grid; c += 32) {
      const double l = *reinterpret_cast<volatile double*>(losses + c);
      if (l < v) { v = l; idx = c; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, v, off);
      const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
      if (ov < v || (ov == v && oi < idx)) { v = ov; idx = oi; }
    }
    if (lane == 0) {
      if (failed || idx == 0x7fffffff) idx = -1;
      best_sh = idx;
      *best_j = idx;
    }
  }
  __syncthreads();
  const int b = best_sh;
  if (b >= 0)
    for (int64_t k = threadIdx.x; k < K; k += kFinThreads) scales[k] = table[static_cast<int64_t>(b) * K + k];
}

// ===================================================================================================
// (5) pack: codes, steps and zeros of W at scales s. One warp covers 1024 in-features (a segment) of one
// row; each lane owns 32 consecutive in-features (4 lanes per group of 128, four code words).
// ===================================================================================================
constexpr int kPackThreads = 256;
constexpr int kPackCols = 32;                    // in-features per lane (4 lanes per group of 128)
constexpr int kPackWarpCols = 32 * kPackCols;    // 1024 in-features (one segment) per warp
constexpr int kPackStages = 4;                   // rows in flight per warp (cp.async ring)
constexpr int kPackStageBytes = kPackWarpCols * 2;                                   // 2 KB
constexpr int kPackScaleBytes = kPackWarpCols * 4;                                   // 4 KB
constexpr int kPackSmemBytes = kPackStages * (kPackThreads / 32) * kPackStageBytes + kPackScaleBytes;  // 68 KB
constexpr int kPackCtasPerSm = 3;

// CTA b owns segment b % segs and, warp w, rows 8 (b / segs) + w, stepping by 8 x (CTAs per segment);
// with fewer CTAs than segments a CTA walks several whole segments. The segment's scales sit once in
// shared memory (16-byte piece j of lane l's 32 at offset 16 (32 j + l): conflict-free) and are read back
// for every row, which keeps registers for three CTAs per SM. Each lane streams its own 64 bytes of the
// next rows through a ring in shared memory with cp.async (up to kPackStages - 1 rows in flight per
// warp, no registers held); a lane only reads back what it copied itself, laid out the same way, so the
// ring needs no synchronisation.
__global__ void __launch_bounds__(kPackThreads, kPackCtasPerSm) quantize_pack_kernel(
    const uint16_t* __restrict__ W, int64_t O, int64_t K, int64_t ldw, const float* __restrict__ scales,
    int exact, uint32_t* __restrict__ codes, float* __restrict__ steps, float* __restrict__ zeros) {
  extern __shared__ __align__(16) uint8_t pack_ring[];
  const int64_t segs = (K + kPackWarpCols - 1) / kPackWarpCols;
  const int64_t ctas = gridDim.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem0 = static_cast<uint32_t>(__cvta_generic_to_shared(pack_ring));
  const uint32_t scl = smem0 + static_cast<uint32_t>(kPackStages * (kPackThreads / 32) * kPackStageBytes) +
                       static_cast<uint32_t>(lane) * 16u;
  const uint32_t ring = smem0 + static_cast<uint32_t>(warp * kPackStages * kPackStageBytes) +
                        static_cast<uint32_t>(lane) * 16u;
  int64_t seg_first, seg_step, row_first, row_step;
  if (ctas >= segs) {
    const int64_t cps = ctas / segs;
    if (static_cast<int64_t>(blockIdx.x) >= cps * segs) return;  // the whole CTA
    seg_first = blockIdx.x % segs;
    seg_step = segs;  // one segment
    row_first = (blockIdx.x / segs) * (kPackThreads / 32) + warp;
    row_step = cps * (kPackThreads / 32);
  } else {
    seg_first = blockIdx.x;
    seg_step = ctas;
    row_first = warp;
    row_step = kPackThreads / 32;
  }
  for (int64_t seg = seg_first; seg < segs; seg += seg_step) {
    const int64_t k0 = seg * kPackWarpCols + static_cast<int64_t>(lane) * kPackCols;
    const bool active = k0 < K;  // K % 128 == 0: 4-lane groups are all active or all idle
    {
      // thread (w, l) stages piece w of lane l's scales (1.0 past K)
      const int64_t kk = seg * kPackWarpCols + static_cast<int64_t>(lane) * kPackCols + 4 * warp;
      const float4 x = kk < K ? __ldg(reinterpret_cast<const float4*>(scales + kk)) : make_float4(1.f, 1.f, 1.f, 1.f);
      __syncthreads();  // the previous segment's scales are no longer read
      asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(scl + static_cast<uint32_t>(warp * 512)),
                   "f"(x.x), "f"(x.y), "f"(x.z), "f"(x.w)
                   : "memory");
      __syncthreads();
    }
    // row i of this warp is o = row_first + i * row_step, staged in slot i % kPackStages
    auto issue = [&](int64_t i) {
      const int64_t o = row_first + i * row_step;
      if (o < O && active) {
        const uint16_t* src = W + o * ldw + k0;
        const uint32_t dst = ring + static_cast<uint32_t>((i % kPackStages) * kPackStageBytes);
#pragma unroll
        for (int j = 0; j < 4; ++j) cp_async_16(dst + static_cast<uint32_t>(j * 512), src + 8 * j, 16u);
      }
      cp_async_commit();  // an empty group keeps the wait arithmetic uniform
    };
#pragma unroll 1
    for (int64_t i = 0; i < kPackStages - 1; ++i) issue(i);
#pragma unroll 1
    for (int64_t i = 0; row_first + i * row_step < O; ++i) {
      const int64_t o = row_first + i * row_step;
      issue(i + kPackStages - 1);  // into the slot read in the previous iteration
      cp_async_wait<kPackStages - 1>();
      uint4 cur[4];
      const uint32_t src = ring + static_cast<uint32_t>((i % kPackStages) * kPackStageBytes);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(cur[j].x), "=r"(cur[j].y), "=r"(cur[j].z), "=r"(cur[j].w)
                     : "r"(src + static_cast<uint32_t>(j * 512))
                     : "memory");
      // w' = RN(w * s) in pairs (elements 2i, 2i+1 of the lane's 32 in-features); the lane's max and min
      // by a tree of three-input min/max (8 partial results of 4 elements each, then 3, then 1)
      uint64_t wp2[kPackCols / 2];
      float px[8], pn[8];
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const uint32_t uu[4] = {cur[v4].x, cur[v4].y, cur[v4].z, cur[v4].w};
        float4 sa, sb;  // scales of elements 8 v4 .. 8 v4 + 7
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(sa.x), "=f"(sa.y), "=f"(sa.z), "=f"(sa.w)
                     : "r"(scl + static_cast<uint32_t>(2 * v4 * 512)));
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(sb.x), "=f"(sb.y), "=f"(sb.z), "=f"(sb.w)
                     : "r"(scl + static_cast<uint32_t>((2 * v4 + 1) * 512)));
        wp2[4 * v4 + 0] = fx2_mul(fx2(bf16_lo(uu[0]), bf16_hi(uu[0])), fx2(sa.x, sa.y));
        wp2[4 * v4 + 1] = fx2_mul(fx2(bf16_lo(uu[1]), bf16_hi(uu[1])), fx2(sa.z, sa.w));
        wp2[4 * v4 + 2] = fx2_mul(fx2(bf16_lo(uu[2]), bf16_hi(uu[2])), fx2(sb.x, sb.y));
        wp2[4 * v4 + 3] = fx2_mul(fx2(bf16_lo(uu[3]), bf16_hi(uu[3])), fx2(sb.z, sb.w));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float a0, b0, a1, b1;
          fx2_split(wp2[4 * v4 + 2 * h], a0, b0);
          fx2_split(wp2[4 * v4 + 2 * h + 1], a1, b1);
          px[2 * v4 + h] = max3f(a0, b0, fmaxf(a1, b1));
          pn[2 * v4 + h] = min3f(a0, b0, fminf(a1, b1));
        }
      }
      float mx = max3f(max3f(px[0], px[1], px[2]), max3f(px[3], px[4], px[5]), fmaxf(px[6], px[7]));
      float mn = min3f(min3f(pn[0], pn[1], pn[2]), min3f(pn[3], pn[4], pn[5]), fminf(pn[6], pn[7]));
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      }
      if (!active) continue;
      const GroupParams g = group_params(mx, mn);
      uint32_t word[4];
      float C = 0.0f;
      bool fast = exact == 0 && fast_group(g, mx, mn, C);
      if (fast) {
        // t = RN(RN(w' * rstep) + C); its low byte is the code; pairs of codes are joined by one
        // integer multiply-add (t1 * 16 + t0: the low byte is c0 + 16 c1, no carry out of it), two
        // pairs by another (p23 * 256 + p01), and the two halves of a word by a byte permute.
        // The tie test |d| < kTieMargin is taken on RN(d^2) < RN(kTieMargin^2), which implies it (RN is
        // monotone), from a paired multiply and one three-input max per pair.
        const uint64_t rs2 = fx2(g.rstep, g.rstep), C2 = fx2(C, C);
        float dq[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t p[4];  // p[e2]: low byte = codes of elements 8w + 2e2 and 8w + 2e2 + 1
          float q0 = 0.0f, q1 = 0.0f;
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const uint64_t qa = fx2_mul(wp2[4 * w + e2], rs2);
            const uint64_t t = fx2_add(qa, C2);
            const uint64_t d = fx2_sub(qa, fx2_sub(t, C2));
            float d0, d1, t0, t1;
            fx2_split(fx2_mul(d, d), d0, d1);
            fx2_split(t, t0, t1);
            if (e2 < 2) q0 = max3f(q0, d0, d1);
            else q1 = max3f(q1, d0, d1);
            p[e2] = __float_as_uint(t1) * 16u + __float_as_uint(t0);
          }
          dq[w] = fmaxf(q0, q1);
          word[w] = __byte_perm(p[1] * 256u + p[0], p[3] * 256u + p[2], 0x5410);
        }
        fast = fmaxf(fmaxf(dq[0], dq[1]), fmaxf(dq[2], dq[3])) < kTieMarginSq;
      }
      if (!fast) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          word[w] = 0u;
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float a, b;
            fx2_split(wp2[(8 * w + e) / 2], a, b);
            word[w] |= static_cast<uint32_t>(code_of(a, g, exact != 0)) << (4 * e);
            word[w] |= static_cast<uint32_t>(code_of(b, g, exact != 0)) << (4 * e + 4);
          }
        }
      }
      __stcs(reinterpret_cast<uint4*>(codes + o * (K / 8) + k0 / 8), make_uint4(word[0], word[1], word[2], word[3]));
      if ((lane & 3) == 0) {
        const int64_t gi = o * (K / 128) + k0 / 128;
        steps[gi] = g.step;
        zeros[gi] = g.zero;
      }
    }
    cp_async_wait<0>();  // nothing of this segment's ring is still being written
  }
}

// ===================================================================================================
// Scale folding: out = bf16(RN32(A op s)) with s per column or per row. 8 elements per thread.
// ===================================================================================================
constexpr int kFoldThreads = 256;

template <bool kColumns>
__global__ void __launch_bounds__(kFoldThreads) scale_fold_kernel(const uint16_t* __restrict__ A, int64_t R,
                                                                  int64_t C, int64_t lda,
                                                                  const float* __restrict__ s, int divide,
                                                                  uint16_t* __restrict__ out, int64_t ldo) {
  const int64_t vec_per_row = C / 8;
  const int64_t total = R * vec_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kFoldThreads) {
    const int64_t r = i / vec_per_row;
    const int64_t c0 = (i - r * vec_per_row) * 8;
    const uint4 u = *reinterpret_cast<const uint4*>(A + r * lda + c0);
    float sv[8];
    if (kColumns) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(s + c0));
      const float4 b = __ldg(reinterpret_cast<const float4*>(s + c0) + 1);
      sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w; sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
    } else {
      const float x = __ldg(s + r);
#pragma unroll
      for (int k = 0; k < 8; ++k) sv[k] = x;
    }
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = bf16_lo(w[k]), hi = bf16_hi(w[k]);
      const float rl = divide ? __fdiv_rn(lo, sv[2 * k]) : __fmul_rn(lo, sv[2 * k]);
      const float rh = divide ? __fdiv_rn(hi, sv[2 * k + 1]) : __fmul_rn(hi, sv[2 * k + 1]);
      const __nv_bfloat162 pr = __floats2bfloat162_rn(rl, rh);
      o[k] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    *reinterpret_cast<uint4*>(out + r * ldo + c0) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ===================================================================================================
// INT8 per-channel quantizer: per-row steps of every candidate, and the INT8 pack.
// ===================================================================================================
constexpr int kRowThreads = 256;  // one warp per (candidate, row)

// rowstep[j][o] = max(RN32(max_k |RN32(w[o,k] * s_j[k])| / 127), 1e-5); rows o >= O get 1.
__global__ void __launch_bounds__(kRowThreads) int8_rowstep_kernel(const uint16_t* __restrict__ W, int64_t O,
                                                                   int64_t O_pad, int64_t K, int64_t ldw,
                                                                   const float* __restrict__ table,
                                                                   float* __restrict__ rowstep) {
  const int64_t o = (static_cast<int64_t>(blockIdx.x) * kRowThreads + threadIdx.x) >> 5;
  const int j = blockIdx.y;
  const int lane = threadIdx.x & 31;
  if (o >= O_pad) return;
  float amax = 0.0f;
  if (o < O) {
    const float* sj = table + static_cast<int64_t>(j) * K;
    for (int64_t k0 = static_cast<int64_t>(lane) * 8; k0 < K; k0 += 256) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(W + o * ldw + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(sj + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(sj + k0) + 1);
      const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
      const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(__fmul_rn(bf16_lo(uu[i]), ss[2 * i])));
        amax = fmaxf(amax, fabsf(__fmul_rn(bf16_hi(uu[i]), ss[2 * i + 1])));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) rowstep[static_cast<int64_t>(j) * O_pad + o] = o < O ? int8_params(amax).step : 1.0f;
}

// One warp per row (grid-stride): the row's max |w'|, then its codes (int8) and step.
__global__ void __launch_bounds__(kRowThreads) quantize_pack_int8_kernel(
    const uint16_t* __restrict__ W, int64_t O, int64_t K, int64_t ldw, const float* __restrict__ scales, int exact,
    int8_t* __restrict__ codes, float* __restrict__ steps) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * kRowThreads) >> 5;
  for (int64_t o = (static_cast<int64_t>(blockIdx.x) * kRowThreads + threadIdx.x) >> 5; o < O; o += warps) {
    float amax = 0.0f;
    for (int64_t k0 = static_cast<int64_t>(lane) * 8; k0 < K; k0 += 256) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(W + o * ldw + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(scales + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(scales + k0) + 1);
      const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
      const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(__fmul_rn(bf16_lo(uu[i]), ss[2 * i])));
        amax = fmaxf(amax, fabsf(__fmul_rn(bf16_hi(uu[i]), ss[2 * i + 1])));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const GroupParams g = int8_params(amax);
    for (int64_t k0 = static_cast<int64_t>(lane) * 8; k0 < K; k0 += 256) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(W + o * ldw + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(scales + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(scales + k0) + 1);
      const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
      const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q0 = static_cast<int>(code_of_int8(__fmul_rn(bf16_lo(uu[i]), ss[2 * i]), g, exact != 0));
        const int q1 = static_cast<int>(code_of_int8(__fmul_rn(bf16_hi(uu[i]), ss[2 * i + 1]), g, exact != 0));
        packed[i / 2] |= (static_cast<uint32_t>(q0) & 0xFFu) << (16 * (i & 1));
        packed[i / 2] |= (static_cast<uint32_t>(q1) & 0xFFu) << (16 * (i & 1) + 8);
      }
      *reinterpret_cast<uint2*>(codes + o * K + k0) = make_uint2(packed[0], packed[1]);
    }
    if (lane == 0) steps[o] = g.step;
  }
}

// One CTA per row (grid-stride), the row held in registers: every thread keeps NV 16-byte pieces of it
// (piece v of thread t = in-features 8 (256 v + t) ..), so W is read once. The row's max |w'| is reduced
// over the CTA, then each thread codes its pieces. K <= 2048 NV.
constexpr int kRowBlock = 256;
template <int NV>
__global__ void __launch_bounds__(kRowBlock) quantize_pack_int8_rows_kernel(
    const uint16_t* __restrict__ W, int64_t O, int64_t K, int64_t ldw, const float* __restrict__ scales, int exact,
    int8_t* __restrict__ codes, float* __restrict__ steps) {
  __shared__ float wmax[kRowBlock / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  for (int64_t o = blockIdx.x; o < O; o += gridDim.x) {
    uint4 u[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int64_t k0 = (static_cast<int64_t>(v) * kRowBlock + t) * 8;
      u[v] = k0 < K ? __ldg(reinterpret_cast<const uint4*>(W + o * ldw + k0)) : make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int64_t k0 = (static_cast<int64_t>(v) * kRowBlock + t) * 8;
      if (k0 < K) {
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(scales + k0));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(scales + k0) + 1);
        const uint32_t uu[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
        const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          amax = fmaxf(amax, fabsf(__fmul_rn(bf16_lo(uu[i]), ss[2 * i])));
          amax = fmaxf(amax, fabsf(__fmul_rn(bf16_hi(uu[i]), ss[2 * i + 1])));
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) wmax[warp] = amax;
    __syncthreads();
    amax = wmax[0];
#pragma unroll
    for (int w = 1; w < kRowBlock / 32; ++w) amax = fmaxf(amax, wmax[w]);
    __syncthreads();  // wmax is rewritten for the next row
    const GroupParams g = int8_params(amax);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int64_t k0 = (static_cast<int64_t>(v) * kRowBlock + t) * 8;
      if (k0 < K) {
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(scales + k0));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(scales + k0) + 1);
        const uint32_t uu[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
        const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q0 = static_cast<int>(code_of_int8(__fmul_rn(bf16_lo(uu[i]), ss[2 * i]), g, exact != 0));
          const int q1 = static_cast<int>(code_of_int8(__fmul_rn(bf16_hi(uu[i]), ss[2 * i + 1]), g, exact != 0));
          packed[i / 2] |= (static_cast<uint32_t>(q0) & 0xFFu) << (16 * (i & 1));
          packed[i / 2] |= (static_cast<uint32_t>(q1) & 0xFFu) << (16 * (i & 1) + 8);
        }
        *reinterpret_cast<uint2*>(codes + o * K + k0) = make_uint2(packed[0], packed[1]);
      }
    }
    if (t == 0) steps[o] = g.step;
  }
}

}  // namespace awq
