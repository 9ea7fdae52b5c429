// Block pooling: mean of every 64-token block of Q, K and V.
//
// Sol-Attn keeps "pooled K/V summaries" per block and scores query blocks
// against key blocks with light query-key scores (Sol-H3 DGX Spark release,
// arex-research 3d0ff631, Sol-Attn bullet of the five optimisations); the
// blocks are 64 tokens (Sol-H3 overview, yanziyuan 171844, "sparse
// attention" paragraph).  The mean is the pooling operator.
//
// HBM-bound: one pass over Q, K, V with 16-byte vector loads, fp32 sums.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sol {

constexpr int kBlock = 64;

struct PoolOut {
  float* qbar_f32;           // [rows/64, D]
  float* kbar_f32;           // [rows/64, D]
  __nv_bfloat16* kbar_bf16;  // [rows/64, D]
  __nv_bfloat16* vbar_bf16;  // [rows/64, D]
};

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], uint4 x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// grid (num_blocks, 3): blockIdx.y selects Q, K or V; 128 threads per CTA,
// one CTA per 64-row block of one tensor.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   const __nv_bfloat16* __restrict__ v,
                                                   PoolOut o) {
  constexpr int kThreadsPerRow = D / 8;                 // 16 B (8 bf16) per thread per row
  constexpr int kRowsPerPass = 128 / kThreadsPerRow;
  constexpr int kPasses = kBlock / kRowsPerPass;
  __shared__ float red[kRowsPerPass][D];

  const int which = blockIdx.y;
  const __nv_bfloat16* src = which == 0 ? q : (which == 1 ? k : v);
  const size_t blk = blockIdx.x;
  const int t = threadIdx.x;
  const int col = (t % kThreadsPerRow) * 8;
  const int r0 = t / kThreadsPerRow;

  const uint4* base = reinterpret_cast<const uint4*>(src + blk * kBlock * D);
  uint4 x[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    x[p] = __ldg(base + ((r0 + p * kRowsPerPass) * D + col) / 8);
  }
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int p = 0; p < kPasses; ++p) add_bf16x8(acc, x[p]);
#pragma unroll
  for (int i = 0; i < 8; ++i) red[r0][col + i] = acc[i];
  __syncthreads();

  for (int c = t; c < D; c += 128) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) s += red[r][c];
    const float mean = s * (1.0f / kBlock);  // exact scaling by a power of two
    const size_t idx = blk * D + c;
    if (which == 0) {
      o.qbar_f32[idx] = mean;
    } else if (which == 1) {
      o.kbar_f32[idx] = mean;
      o.kbar_bf16[idx] = __float2bfloat16_rn(mean);
    } else {
      o.vbar_bf16[idx] = __float2bfloat16_rn(mean);
    }
  }
}

// The same pooling for E4M3 inputs (8-bit path; D = 128, one 128-byte row per
// token).  Values are decoded exactly to fp32 and summed in fp32.  The fp32
// means for the router are those of the real values (raw mean times the
// tensor's scale); the 8-bit means for the correction MMA stay in the raw
// domain of their tensor, rounded to E4M3 (nearest even, saturating), so the
// MMA applies the same scales to them as to the exact keys and values.
struct PoolOutE4M3 {
  float* qbar_f32;   // [rows/64, D], real domain
  float* kbar_f32;   // [rows/64, D], real domain
  uint8_t* kbar_e4m3;  // [rows/64, D], raw domain of k
  uint8_t* vbar_e4m3;  // [rows/64, D], raw domain of v
  float q_scale, k_scale;
};

// grid (num_blocks, 3): blockIdx.y selects Q, K or V; 128 threads per CTA.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel_e4m3(const uint8_t* __restrict__ q,
                                                        const uint8_t* __restrict__ k,
                                                        const uint8_t* __restrict__ v,
                                                        PoolOutE4M3 o) {
  constexpr int kThreadsPerRow = D / 16;               // 16 B (16 values) per thread per row
  constexpr int kRowsPerPass = 128 / kThreadsPerRow;
  constexpr int kPasses = kBlock / kRowsPerPass;
  __shared__ float red[kRowsPerPass][D];

  const int which = blockIdx.y;
  const uint8_t* src = which == 0 ? q : (which == 1 ? k : v);
  const size_t blk = blockIdx.x;
  const int t = threadIdx.x;
  const int col = (t % kThreadsPerRow) * 16;
  const int r0 = t / kThreadsPerRow;

  const uint4* base = reinterpret_cast<const uint4*>(src + blk * kBlock * D);
  uint4 x[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) x[p] = __ldg(base + ((r0 + p * kRowsPerPass) * D + col) / 16);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const uint32_t w[4] = {x[p].x, x[p].y, x[p].z, x[p].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a, b, c, d;
      unpack_e4m3x2(static_cast<uint16_t>(w[i] & 0xFFFFu), a, b);
      unpack_e4m3x2(static_cast<uint16_t>(w[i] >> 16), c, d);
      acc[4 * i] += a;
      acc[4 * i + 1] += b;
      acc[4 * i + 2] += c;
      acc[4 * i + 3] += d;
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) red[r0][col + i] = acc[i];
  __syncthreads();

  for (int c = t; c < D; c += 128) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) s += red[r][c];
    const float mean = s * (1.0f / kBlock);  // raw-domain mean (exact scaling by a power of two)
    const size_t idx = blk * D + c;
    if (which == 0) {
      o.qbar_f32[idx] = mean * o.q_scale;
    } else if (which == 1) {
      o.kbar_f32[idx] = mean * o.k_scale;
      o.kbar_e4m3[idx] = static_cast<uint8_t>(pack_e4m3x4(mean, 0.f, 0.f, 0.f) & 0xFFu);
    } else {
      o.vbar_e4m3[idx] = static_cast<uint8_t>(pack_e4m3x4(mean, 0.f, 0.f, 0.f) & 0xFFu);
    }
  }
}

}  // namespace sol
