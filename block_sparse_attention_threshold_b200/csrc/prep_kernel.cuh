// QKNorm + partial RoPE of Q and K with the block pooling fused in.
//
// The pages list "QKNorm + partial RoPE" among the fused chains whose
// intermediates stay in registers or on chip ("MiniMax 官宣 NVIDIA Sol 团队 H3
// 加速", arex-research 2a2a70ca, section "speed-up comes from stacking every
// stage of the pipeline", fused-operators item; kocpc.com.tw report of the
// same release, section "技術組成"), and Sol-Attn needs pooled summaries of
// the normalised, rotated Q and K.  This kernel writes Q and K after the chain
// and, in the same pass, the pooled workspace that the attention step reads,
// so no separate pooling pass re-reads them from HBM.
//
// The pages name the chain only; the readings:
//  * QKNorm = RMSNorm over the head dimension with a per-dimension weight:
//    y = x * rsqrt(mean(x^2) + eps) * w;
//  * partial RoPE rotates the first R dimensions, pairing i with i + R/2 for
//    i < R/2 by pos * base^(-2 i / R); pos = token index in the sequence;
//  * the pooled means are those of the written bf16 values, summed in the
//    same order as the standalone pooling kernel, so both give the same bits.
//
// HBM-bound: one pass over Q, K (and V when pooling) with 16-byte accesses.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "pool_kernel.cuh"

namespace sol {

struct PrepParams {
  const __nv_bfloat16* q_in;
  const __nv_bfloat16* k_in;
  const __nv_bfloat16* v;      // read only when pooling
  const float* wq;             // [D] QKNorm weights
  const float* wk;             // [D]
  __nv_bfloat16* q_out;        // [rows, D]
  __nv_bfloat16* k_out;        // [rows, D]
  PoolOut pool;                // used only when pooling
  int M;                       // blocks per sequence, N / 64
  int rope_dims;               // R: 0, or 16 * 2^k <= D
  float eps;
  double inv_freq[64];         // base^(-2 i / R) for i < R/2, computed on the host in double
};

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&h);
}

// grid (B*H*M, kPool ? 3 : 2): blockIdx.y selects Q, K or V; 128 threads,
// one CTA per 64-row block of one tensor, laid out as in pool_kernel.
template <int D, bool kPool>
__global__ void __launch_bounds__(128) prep_kernel(const PrepParams p) {
  constexpr int kThreadsPerRow = D / 8;  // 16 B (8 bf16) per thread per row
  constexpr int kRowsPerPass = 128 / kThreadsPerRow;
  constexpr int kPasses = kBlock / kRowsPerPass;
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  __shared__ float red[kPool ? kRowsPerPass : 1][kPool ? D : 1];

  const int which = blockIdx.y;
  const size_t blk = blockIdx.x;
  const int t = threadIdx.x;
  const int col = (t % kThreadsPerRow) * 8;
  const int r0 = t / kThreadsPerRow;
  const __nv_bfloat16* src = which == 0 ? p.q_in : (which == 1 ? p.k_in : p.v);
  const uint4* in = reinterpret_cast<const uint4*>(src + blk * kBlock * D);
  uint4 x[kPasses];
#pragma unroll
  for (int s = 0; s < kPasses; ++s) x[s] = __ldg(in + ((r0 + s * kRowsPerPass) * D + col) / 8);

  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (which < 2) {
    const float* wsrc = which == 0 ? p.wq : p.wk;
    float w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = __ldg(wsrc + col + i);
    const int R = p.rope_dims, half = R / 2;
    const bool rot = col < R;        // this thread's 8 dimensions are rotated
    const bool first = col < half;   // ... as the first members of their pairs
    uint4* out = reinterpret_cast<uint4*>((which == 0 ? p.q_out : p.k_out) + blk * kBlock * D);
    const int pos0 = static_cast<int>(blk % static_cast<size_t>(p.M)) * kBlock;
    // cos / sin of this thread's 8 angles at its first row, and of the step
    // to its next row (kRowsPerPass positions on).  The angle is formed and
    // reduced to [-pi, pi] in double, so positions up to 2^17 keep their
    // precision; later rows advance by the step rotation in fp32 (at most
    // kPasses - 1 steps).
    float cs[8], sn[8], cstep[8], sstep[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cs[i] = 1.f;
      sn[i] = 0.f;
      cstep[i] = 1.f;
      sstep[i] = 0.f;
      if (rot) {
        const double th = p.inv_freq[(first ? col : col - half) + i];
        double a = static_cast<double>(pos0 + r0) * th;
        a -= kTwoPi * rint(a * (1.0 / kTwoPi));
        sincosf(static_cast<float>(a), &sn[i], &cs[i]);
        double b = kRowsPerPass * th;
        b -= kTwoPi * rint(b * (1.0 / kTwoPi));
        sincosf(static_cast<float>(b), &sstep[i], &cstep[i]);
      }
    }
#pragma unroll
    for (int s = 0; s < kPasses; ++s) {
      const int r = r0 + s * kRowsPerPass;
      const uint32_t wd[4] = {x[s].x, x[s].y, x[s].z, x[s].w};
      float f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(wd[i] << 16);
        f[2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
      }
      // RMSNorm: the row's sum of squares over its kThreadsPerRow lanes.
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
#pragma unroll
      for (int o = kThreadsPerRow / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      const float inv = rsqrtf(ss * (1.0f / D) + p.eps);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = f[i] * inv * w[i];
      // Partial RoPE: the partner dimensions (i +- R/2) sit R/16 lanes away.
      if (R > 0) {
        float g[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = __shfl_xor_sync(0xFFFFFFFFu, f[i], R / 16);
        if (rot) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            f[i] = first ? fmaf(f[i], cs[i], -g[i] * sn[i]) : fmaf(g[i], sn[i], f[i] * cs[i]);
            // advance to this thread's next row
            const float c2 = fmaf(cs[i], cstep[i], -sn[i] * sstep[i]);
            sn[i] = fmaf(sn[i], cstep[i], cs[i] * sstep[i]);
            cs[i] = c2;
          }
        }
      }
      uint4 o;
      o.x = bf16x2_rn(f[0], f[1]);
      o.y = bf16x2_rn(f[2], f[3]);
      o.z = bf16x2_rn(f[4], f[5]);
      o.w = bf16x2_rn(f[6], f[7]);
      out[(r * D + col) / 8] = o;
      if constexpr (kPool) add_bf16x8(acc, o);
    }
  } else if constexpr (kPool) {
#pragma unroll
    for (int s = 0; s < kPasses; ++s) add_bf16x8(acc, x[s]);
  }

  if constexpr (kPool) {
    // Same reduction order as pool_kernel: per-thread sums over the passes,
    // then the row groups in order.
#pragma unroll
    for (int i = 0; i < 8; ++i) red[r0][col + i] = acc[i];
    __syncthreads();
    for (int c = t; c < D; c += 128) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < kRowsPerPass; ++r) s += red[r][c];
      const float mean = s * (1.0f / kBlock);
      const size_t idx = blk * D + c;
      if (which == 0) {
        p.pool.qbar_f32[idx] = mean;
      } else if (which == 1) {
        p.pool.kbar_f32[idx] = mean;
        p.pool.kbar_bf16[idx] = __float2bfloat16_rn(mean);
      } else {
        p.pool.vbar_bf16[idx] = __float2bfloat16_rn(mean);
      }
    }
  }
}

}  // namespace sol
