// Fused Sol-Attn forward on sm_100a: routing, exact attention over the kept
// key blocks and the pooled correction of the skipped ones, in one online
// softmax.
//
// What it computes (the pages give prose only):
//  * 64-token blocks; each query block scores its pooled query against the
//    pooled keys and keeps the key blocks whose score is at least
//    mean + tau * std of that block's scores ("MiniMax 官宣 NVIDIA Sol 团队 H3
//    加速", arex-research 2a2a70ca, section "speed-up comes from stacking every
//    stage of the pipeline", Sol-Attn item; Sol-H3 overview, yanziyuan 171844,
//    "sparse attention" paragraph);
//  * kept blocks take exact softmax attention, skipped blocks are corrected
//    from pooled K/V summaries, and routing, sparse compute and correction
//    share one online softmax with no score map or routing index tensor
//    written out (Sol-H3 DGX Spark release, arex-research 3d0ff631, Sol-Attn
//    bullet);
//  * the correction is the zeroth-order term of the "Taylor approximation" of
//    rejected blocks ("MiniMax 官推背书 Sol Engine", arex-research 647c3193,
//    section "3.95x near-lossless"): logit scale * q.kbar_j + ln 64 with value
//    vbar_j;
//  * the text | cond | audio prefix is always exact (yanziyuan 171844,
//    "safety rail" paragraph): prefix query blocks attend densely, prefix key
//    blocks are always kept.
//
// Structure of one CTA (one 128-row query tile = query blocks 2t and 2t+1):
//  warp 0     TMA producer: Q tile, then per stage a 128-key K tile and V tile
//             (two kept 64-key blocks, possibly far apart, or 128 pooled keys);
//  warp 1     tcgen05 issuer: S = Q K^T into TMEM, then O += P V with P read
//             from TMEM (P overwrites S in place as bf16);
//  warps 2-5  router (scores, mean/std, keep bits in shared memory), then
//             online softmax (one TMEM lane = one query row), conditional O
//             rescale, and the epilogue O / l -> bf16.
// The tile visits the union of its two query blocks' kept sets; a row whose
// block did not keep a visited key block masks it out and gets that block's
// pooled correction instead.  Two CTAs share an SM (TMEM 2 x 256 columns),
// so one CTA's softmax overlaps the other's MMAs.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sol {

constexpr int kTileM = 128;     // query rows per CTA (two 64-token blocks)
constexpr int kTileN = 128;     // keys per stage
constexpr int kMaxBlocks = 4096;  // largest M = N / 64 the router supports
constexpr int kMaskWords = kMaxBlocks / 32;
constexpr int kThreads = 192;
constexpr float kLog2Block = 6.0f;        // log2(64): the ln c_j bias in log2 units
constexpr float kRescaleSlack = 8.0f;     // keep a stale max while the new one is <= 2^8 larger

// Device error word: 0 = fine, else the site of the first timed-out wait.
__device__ int g_sol_attn_error = 0;

struct AttnParams {
  int B, H, N, M, P;         // M = N / 64 blocks, P = prefix_len / 64
  int tiles_per_head;        // ceil(M / 2)
  float tau;                 // may be +-inf
  float scale;               // softmax scale (also the score scale)
  float scale_log2;          // scale * log2(e)
  const float* qbar;         // [B*H*M, D] fp32
  const float* kbar;         // [B*H*M, D] fp32
  __nv_bfloat16* out;        // [B*H*N, D]
  uint32_t* debug_mask;      // [B*H*M, ceil(M/32)] or null
  unsigned long long* kept_pairs;   // or null
  unsigned long long* exact_pairs;  // or null
  uint64_t timeout_ns;
  int skip_first_k_arrival;  // test hook: producer never loads stage 0's K tile
};

template <int D>
struct SmemPlan {
  static constexpr int kTileBytes = kTileM * D * 2;  // 128 rows x D bf16
  static constexpr int kChunkBytes = kTileM * 128;   // one 64-column chunk of a 128-row tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kMaskA = kV + kTileBytes;
  static constexpr int kMaskB = kMaskA + kMaskWords * 4;
  static constexpr int kMaskU = kMaskB + kMaskWords * 4;
  static constexpr int kQbar = kMaskU + kMaskWords * 4;  // 2 x D floats
  static constexpr int kRed = kQbar + 2 * D * 4;         // 32 floats
  static constexpr int kBars = kRed + 32 * 4;            // 10 mbarriers
  static constexpr int kMisc = kBars + 10 * 8;           // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;           // room to align the base to 1 KB
  static_assert(2 * kMaxBlocks * 4 <= 2 * kTileBytes || D < 128, "score scratch must fit in K+V");
};

enum BarId { kBarQ = 0, kBarKFull, kBarKEmpty, kBarVFull, kBarVEmpty, kBarSFull, kBarPFull,
             kBarOFull, kBarDrain };

__device__ __forceinline__ bool mask_bit(const uint32_t* m, int j) {
  return (m[j >> 5] >> (j & 31)) & 1u;
}

// Next set bit of `m` at or after `j`, or -1 (m has `nw` words).
__device__ __forceinline__ int next_bit(const uint32_t* m, int j, int nw) {
  int w = j >> 5;
  if (w >= nw) return -1;
  uint32_t bits = m[w] & (0xFFFFFFFFu << (j & 31));
  while (bits == 0) {
    if (++w >= nw) return -1;
    bits = m[w];
  }
  return (w << 5) + __ffs(bits) - 1;
}

// One pass over the work of a tile.  Exact stages pair up the kept blocks of
// the union mask in increasing order (j1 = -1 when the count is odd);
// correction stages cover 128 pooled keys [128c, 128c + 128) that hold at
// least one video block skipped by either query block.
struct Stage {
  int j0, j1;     // exact: key blocks; correction: j0 = tile index c, j1 = -2
  bool corr;
  __device__ __forceinline__ int nkeys() const { return (corr || j1 >= 0) ? 128 : 64; }
};

struct StageIter {
  int j = 0;
  int c = 0;
  __device__ __forceinline__ bool next(Stage& s, const uint32_t* mU, const uint32_t* mA,
                                       const uint32_t* mB, int M, int P, bool dense) {
    const int nw = (M + 31) >> 5;
    if (j < M) {
      const int j0 = next_bit(mU, j, nw);
      if (j0 >= 0 && j0 < M) {
        int j1 = next_bit(mU, j0 + 1, nw);
        if (j1 >= M) j1 = -1;
        s.j0 = j0;
        s.j1 = j1;
        s.corr = false;
        j = j1 < 0 ? M : j1 + 1;
        return true;
      }
      j = M;
    }
    if (dense) return false;
    const int nc = (M + 127) >> 7;
    while (c < nc) {
      const int cc = c++;
      bool any = false;
      for (int w = cc * 4; w < cc * 4 + 4 && w < nw; ++w) {
        uint32_t video = 0xFFFFFFFFu;
        const int lo = w * 32;
        if (lo + 32 <= P) video = 0;
        else if (lo < P) video = 0xFFFFFFFFu << (P - lo);
        if (lo + 32 > M) video &= (M - lo >= 32) ? 0xFFFFFFFFu : ((1u << (M - lo)) - 1u);
        if (((~mA[w]) | (~mB[w])) & video) { any = true; break; }
      }
      if (any) {
        s.j0 = cc;
        s.j1 = -2;
        s.corr = true;
        return true;
      }
    }
    return false;
  }
};

// Block-wide (128 softmax threads, named barrier 1) sum of two values.
__device__ __forceinline__ void sm_reduce2(float& a, float& b, float* red, int st) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
  }
  named_bar_sync(1, 128);
  if ((st & 31) == 0) {
    red[(st >> 5) * 2] = a;
    red[(st >> 5) * 2 + 1] = b;
  }
  named_bar_sync(1, 128);
  a = red[0] + red[2] + red[4] + red[6];
  b = red[1] + red[3] + red[5] + red[7];
}

__device__ __forceinline__ void sm_reduce_minmax(float& mn_a, float& mx_a, float& mn_b, float& mx_b,
                                                 float* red, int st) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn_a = fminf(mn_a, __shfl_xor_sync(0xFFFFFFFFu, mn_a, o));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xFFFFFFFFu, mx_a, o));
    mn_b = fminf(mn_b, __shfl_xor_sync(0xFFFFFFFFu, mn_b, o));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xFFFFFFFFu, mx_b, o));
  }
  named_bar_sync(1, 128);
  if ((st & 31) == 0) {
    red[16 + (st >> 5) * 4 + 0] = mn_a;
    red[16 + (st >> 5) * 4 + 1] = mx_a;
    red[16 + (st >> 5) * 4 + 2] = mn_b;
    red[16 + (st >> 5) * 4 + 3] = mx_b;
  }
  named_bar_sync(1, 128);
  mn_a = fminf(fminf(red[16], red[20]), fminf(red[24], red[28]));
  mx_a = fmaxf(fmaxf(red[17], red[21]), fmaxf(red[25], red[29]));
  mn_b = fminf(fminf(red[18], red[22]), fminf(red[26], red[30]));
  mx_b = fmaxf(fmaxf(red[19], red[23]), fmaxf(red[27], red[31]));
}

// Router: pooled scores of query blocks iA, iB against every video key
// block, population mean/std, threshold, keep bits.  Runs on the 128
// softmax threads; scores live in the (not yet used) K/V staging buffers.
template <int D>
__device__ __forceinline__ void route_tile(const AttnParams& p, int bh, int iA, int iB, bool hasB,
                                           uint8_t* smem, int st) {
  using L = SmemPlan<D>;
  uint32_t* mA = reinterpret_cast<uint32_t*>(smem + L::kMaskA);
  uint32_t* mB = reinterpret_cast<uint32_t*>(smem + L::kMaskB);
  float* sq = reinterpret_cast<float*>(smem + L::kQbar);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* sc = reinterpret_cast<float*>(smem + L::kK);  // [2][kMaxBlocks]
  const int M = p.M, P = p.P, nv = M - P;
  const int nw = (M + 31) >> 5;
  const bool videoA = iA >= P, videoB = hasB && iB >= P;

  if ((videoA || videoB) && nv > 0) {
    const float* qa = p.qbar + (static_cast<size_t>(bh) * M + iA) * D;
    const float* qb = p.qbar + (static_cast<size_t>(bh) * M + (hasB ? iB : iA)) * D;
    for (int d = st; d < D; d += 128) {
      sq[d] = qa[d];
      sq[D + d] = qb[d];
    }
    named_bar_sync(1, 128);
    // One thread per video key block: 16-byte loads of its pooled key row.
    const float* kb = p.kbar + static_cast<size_t>(bh) * M * D;
    for (int j = P + st; j < M; j += 128) {
      const float4* row = reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D);
      float da = 0.f, db = 0.f;
#pragma unroll 8
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = __ldg(row + d4);
        const float4 a = reinterpret_cast<const float4*>(sq)[d4];
        const float4 b = reinterpret_cast<const float4*>(sq + D)[d4];
        da = fmaf(a.x, kv.x, da); da = fmaf(a.y, kv.y, da);
        da = fmaf(a.z, kv.z, da); da = fmaf(a.w, kv.w, da);
        db = fmaf(b.x, kv.x, db); db = fmaf(b.y, kv.y, db);
        db = fmaf(b.z, kv.z, db); db = fmaf(b.w, kv.w, db);
      }
      sc[j - P] = da * p.scale;
      sc[kMaxBlocks + j - P] = db * p.scale;
    }
    named_bar_sync(1, 128);
    // Pass 1: mean (and exact-equality check through min/max).
    float sa = 0.f, sb = 0.f;
    float mna = INFINITY, mxa = -INFINITY, mnb = INFINITY, mxb = -INFINITY;
    for (int j = st; j < nv; j += 128) {
      const float a = sc[j], b = sc[kMaxBlocks + j];
      sa += a; sb += b;
      mna = fminf(mna, a); mxa = fmaxf(mxa, a);
      mnb = fminf(mnb, b); mxb = fmaxf(mxb, b);
    }
    sm_reduce2(sa, sb, red, st);
    sm_reduce_minmax(mna, mxa, mnb, mxb, red, st);
    const float mua = sa / nv, mub = sb / nv;
    // Pass 2: population variance about the mean.
    float va = 0.f, vb = 0.f;
    for (int j = st; j < nv; j += 128) {
      const float a = sc[j] - mua, b = sc[kMaxBlocks + j] - mub;
      va = fmaf(a, a, va);
      vb = fmaf(b, b, vb);
    }
    named_bar_sync(1, 128);  // everyone has read red[] of the previous reduction
    sm_reduce2(va, vb, red, st);
    const float sda = (mna == mxa) ? 0.f : sqrtf(va / nv);
    const float sdb = (mnb == mxb) ? 0.f : sqrtf(vb / nv);
    const bool allA = (p.tau == -INFINITY) || sda == 0.f;
    const bool allB = (p.tau == -INFINITY) || sdb == 0.f;
    const float thrA = mua + p.tau * sda;
    const float thrB = mub + p.tau * sdb;
    // Keep bits, one 32-block word per warp iteration.
    const int lane = st & 31, wq = st >> 5;
    for (int w = wq; w < nw; w += 4) {
      const int j = w * 32 + lane;
      bool ka = true, kb2 = true;
      if (j >= M) {
        ka = kb2 = false;
      } else if (j >= P) {
        if (videoA && !allA) ka = sc[j - P] >= thrA;
        if (videoB && !allB) kb2 = sc[kMaxBlocks + j - P] >= thrB;
      }
      const uint32_t wa = __ballot_sync(0xFFFFFFFFu, ka);
      const uint32_t wb = __ballot_sync(0xFFFFFFFFu, kb2);
      if (lane == 0) {
        mA[w] = wa;
        mB[w] = hasB ? wb : wa;
      }
    }
  } else {
    // Prefix query blocks (or no video keys): every block kept.
    for (int w = st; w < nw; w += 128) {
      const int lo = w * 32;
      const uint32_t full = (M - lo >= 32) ? 0xFFFFFFFFu : ((1u << (M - lo)) - 1u);
      mA[w] = full;
      mB[w] = full;
    }
  }
}

template <int D, bool kDense>
__global__ void __launch_bounds__(kThreads, 2)
    sol_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKb,
                        const __grid_constant__ CUtensorMap tmVb, const AttnParams p) {
  using L = SmemPlan<D>;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kTmemCols = 256;
  constexpr uint32_t kColS = 0, kColO = 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  uint32_t* mA = reinterpret_cast<uint32_t*>(smem + L::kMaskA);
  uint32_t* mB = reinterpret_cast<uint32_t*>(smem + L::kMaskB);
  uint32_t* mU = reinterpret_cast<uint32_t*>(smem + L::kMaskU);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.tiles_per_head;
  const int qt = blockIdx.x % p.tiles_per_head;
  const int M = p.M, P = p.P;
  const int iA = 2 * qt, iB = 2 * qt + 1;
  const bool hasB = iB < M;
  const int nw = (M + 31) >> 5;
  int* err = &g_sol_attn_error;

  if (tid == 0) {
    mbar_init(&bars[kBarQ], 1);
    mbar_init(&bars[kBarKFull], 1);
    mbar_init(&bars[kBarKEmpty], 1);
    mbar_init(&bars[kBarVFull], 1);
    mbar_init(&bars[kBarVEmpty], 1);
    mbar_init(&bars[kBarSFull], 1);
    mbar_init(&bars[kBarPFull], 128);
    mbar_init(&bars[kBarOFull], 1);
    mbar_init(&bars[kBarDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Q tile first: it does not depend on the routing.
  const size_t row0 = static_cast<size_t>(bh) * p.N + static_cast<size_t>(qt) * kTileM;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(&bars[kBarQ], kTileM * D * 2);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        tma_load_2d(sQ + c * L::kChunkBytes + h * 64 * 128, &tmQ, &bars[kBarQ], c * 64,
                    static_cast<int>(row0 + h * 64));
  }

  // Routing (softmax warps), or the all-kept mask of the dense kernel.
  if (warp >= 2) {
    const int st = tid - 64;
    if (kDense) {
      for (int w = st; w < nw; w += 128) {
        const int lo = w * 32;
        const uint32_t full = (M - lo >= 32) ? 0xFFFFFFFFu : ((1u << (M - lo)) - 1u);
        mA[w] = full;
        mB[w] = full;
      }
    } else {
      route_tile<D>(p, bh, iA, iB, hasB, smem, st);
    }
    named_bar_sync(1, 128);
    for (int w = st; w < nw; w += 128) mU[w] = mA[w] | mB[w];
    if (!kDense && (p.debug_mask != nullptr || p.kept_pairs != nullptr || p.exact_pairs != nullptr)) {
      unsigned long long kept = 0, uni = 0;
      for (int w = st; w < nw; w += 128) {
        kept += __popc(mA[w]) + (hasB ? __popc(mB[w]) : 0);
        uni += __popc(mA[w] | mB[w]) * (hasB ? 2 : 1);
        if (p.debug_mask != nullptr) {
          p.debug_mask[(static_cast<size_t>(bh) * M + iA) * nw + w] = mA[w];
          if (hasB) p.debug_mask[(static_cast<size_t>(bh) * M + iB) * nw + w] = mB[w];
        }
      }
      if (p.kept_pairs != nullptr && kept) atomicAdd(p.kept_pairs, kept);
      if (p.exact_pairs != nullptr && uni) atomicAdd(p.exact_pairs, uni);
    }
    fence_proxy_async_smem();  // scores were written to K/V staging by generic stores
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const size_t krow_head = static_cast<size_t>(bh) * p.N;
      const size_t prow_head = static_cast<size_t>(bh) * M;
      StageIter it;
      Stage s;
      int n = 0;
      bool ok = true;
      while (ok && it.next(s, mU, mA, mB, M, P, kDense)) {
        const int nhalves = s.corr ? 2 : (s.j1 >= 0 ? 2 : 1);
        const uint32_t bytes = nhalves * kChunks * 64 * 128;
        const CUtensorMap* mk = s.corr ? &tmKb : &tmK;
        const CUtensorMap* mv = s.corr ? &tmVb : &tmV;
        int r[2];
        if (s.corr) {
          r[0] = static_cast<int>(prow_head + s.j0 * 128);
          r[1] = r[0] + 64;
        } else {
          r[0] = static_cast<int>(krow_head + static_cast<size_t>(s.j0) * 64);
          r[1] = static_cast<int>(krow_head + static_cast<size_t>(s.j1 < 0 ? 0 : s.j1) * 64);
        }
        if (n > 0) ok = mbar_wait(&bars[kBarKEmpty], (n - 1) & 1, abort_flag, err, 1, p.timeout_ns);
        if (!ok) break;
        if (!(p.skip_first_k_arrival && n == 0)) {
          mbar_arrive_expect_tx(&bars[kBarKFull], bytes);
          for (int h = 0; h < nhalves; ++h)
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(sK + c * L::kChunkBytes + h * 64 * 128, mk, &bars[kBarKFull], c * 64, r[h]);
        }
        if (n > 0) ok = mbar_wait(&bars[kBarVEmpty], (n - 1) & 1, abort_flag, err, 2, p.timeout_ns);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars[kBarVFull], bytes);
        for (int h = 0; h < nhalves; ++h)
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(sV + c * L::kChunkBytes + h * 64 * 128, mv, &bars[kBarVFull], c * 64, r[h]);
        ++n;
      }
      if (!ok || *abort_flag) {
        // Let loads already issued land before the CTA's shared memory is released.
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) { }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint32_t idesc_pv = idesc_bf16_f32(kTileM, D, true);
      bool ok = mbar_wait(&bars[kBarQ], 0, abort_flag, err, 3, p.timeout_ns);
      StageIter it;
      Stage s;
      int n = 0;
      while (ok && it.next(s, mU, mA, mB, M, P, kDense)) {
        const int nk = s.nkeys();
        ok = mbar_wait(&bars[kBarKFull], n & 1, abort_flag, err, 4, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t idesc_qk = idesc_bf16_f32(kTileM, nk, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColS, sdesc_sw128(sQa + off, 16, 1024), sdesc_sw128(sKa + off, 16, 1024),
                      idesc_qk, kk > 0);
        }
        mma_commit(&bars[kBarSFull]);
        mma_commit(&bars[kBarKEmpty]);
        ok = mbar_wait(&bars[kBarPFull], n & 1, abort_flag, err, 5, p.timeout_ns);
        if (ok) ok = mbar_wait(&bars[kBarVFull], n & 1, abort_flag, err, 6, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < nk / 16; ++kk) {
          mma_bf16_ts(tmem + kColO, tmem + kColS + kk * 8,
                      sdesc_sw128(sVa + kk * 16 * 128, L::kChunkBytes, 1024), idesc_pv,
                      (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kBarVEmpty]);
        ++n;
      }
      mma_commit(&bars[kBarOFull]);
      mma_commit(&bars[kBarDrain]);
      // Drain: the CTA must not free TMEM while MMAs are still running.
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&bars[kBarDrain], 0) && global_timer_ns() - t0 < 2000000000ull) { }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int sp = warp & 3;               // TMEM sub-partition of this warp
    const int r = sp * 32 + lane;          // query row within the tile
    const uint32_t* rowmask = r < 64 ? mA : mB;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sp * 32) << 16);
    float m = -INFINITY, l = 0.f;
    StageIter it;
    Stage s;
    int n = 0;
    bool ok = true;
    while (it.next(s, mU, mA, mB, M, P, kDense)) {
      ok = mbar_wait(&bars[kBarSFull], n & 1, abort_flag, err, 7, p.timeout_ns);
      if (!ok) break;
      tc_fence_after();
      const int nch = s.nkeys() / 32;  // 32-key chunks in this stage (2 or 4)
      // S row -> registers (all of it before P overwrites it in place).
      uint32_t sv[4][32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        if (ch < nch) tmem_ld32(lane_addr + kColS + ch * 32, sv[ch]);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        if (ch < nch) tmem_ld_wait(sv[ch]);
      // Scaled, masked logits in log2 units, written back over sv.
      float tmax = -INFINITY;
      if (!s.corr) {
        const bool k0 = mask_bit(rowmask, s.j0);
        const bool k1 = s.j1 >= 0 && mask_bit(rowmask, s.j1);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if (ch < nch) {
            const bool keep = ch < 2 ? k0 : k1;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float xv = keep ? __uint_as_float(sv[ch][c]) * p.scale_log2 : -INFINITY;
              sv[ch][c] = __float_as_uint(xv);
              tmax = fmaxf(tmax, xv);
            }
          }
        }
      } else {
        const int jb = s.j0 * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          // pooled blocks of this chunk that this row must use: video, in range, skipped
          const int lo = jb + ch * 32;
          uint32_t video = 0xFFFFFFFFu;
          if (lo >= M) {
            video = 0;
          } else {
            if (lo + 32 <= P) video = 0;
            else if (lo < P) video = 0xFFFFFFFFu << (P - lo);
            if (M - lo < 32) video &= (1u << (M - lo)) - 1u;
          }
          const uint32_t use = video ? (~rowmask[lo >> 5] & video) : 0u;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float xv = ((use >> c) & 1u) ? fmaf(__uint_as_float(sv[ch][c]), p.scale_log2, kLog2Block)
                                               : -INFINITY;
            sv[ch][c] = __float_as_uint(xv);
            tmax = fmaxf(tmax, xv);
          }
        }
      }
      // Online softmax with a stale max: rescale O only when the running max
      // grows by more than 2^8; m, l and O always share the same reference.
      // tcgen05.ld/st are warp-collective, so the O pass runs when any row of
      // the warp needs it (alpha = 1 for the others).
      const bool need = (m != -INFINITY) && (tmax > m + kRescaleSlack);
      if (__any_sync(0xFFFFFFFFu, need)) {
        const float alpha = need ? fast_exp2(m - tmax) : 1.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + c0, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(lane_addr + kColO + c0, o);
        }
        l *= alpha;
      }
      if (need || (m == -INFINITY && tmax > m)) m = tmax;
      const float mref = (m == -INFINITY) ? 0.f : m;
      // P = 2^(x - m) as bf16 pairs, 16 TMEM columns per 32-key chunk.
      float rs = 0.f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        if (ch < nch) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float p0 = fast_exp2(__uint_as_float(sv[ch][2 * c]) - mref);
            const float p1 = fast_exp2(__uint_as_float(sv[ch][2 * c + 1]) - mref);
            rs += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st16(lane_addr + kColS + ch * 16, pk);
        }
      }
      l += rs;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[kBarPFull]);
      ++n;
    }
    // Epilogue: out = O / l.
    if (ok) ok = mbar_wait(&bars[kBarOFull], 0, abort_flag, err, 8, p.timeout_ns);
    if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const int grow = qt * kTileM + r;
      __nv_bfloat16* dst = p.out + (static_cast<size_t>(bh) * p.N + grow) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kColO + c0, o);
        tmem_ld_wait(o);
        if (grow < p.N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[c + 0]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l);
            d4[c / 8] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sol
