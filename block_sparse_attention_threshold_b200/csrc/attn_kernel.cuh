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
//  warp 0     TMA producer: the Q tile, then per stage one 64-key block of K
//             and one of V (a kept block, or 64 pooled keys for the
//             correction) into separate 2-deep K and V rings, so the next K
//             lands while the current block is still in the softmax;
//  warp 1     tcgen05 issuer: S = Q K^T into one of two TMEM S buffers, so the
//             next block's scores are computed while the softmax works on the
//             current one; then O += P V with P read from TMEM (P overwrites
//             its S buffer in place as bf16);
//  warps 2-5  online softmax (one TMEM lane = one query row), conditional O
//             rescale, and the epilogue O / l -> bf16.
//  all warps  route first (pooled scores, mean/std, keep bits in shared
//             memory); the two pooled queries are loaded at kernel entry.
// TMEM per CTA: S0 (64 columns) | S1 (64) | O (D) in 256 columns, so two
// CTAs share an SM.
// Grid: one CTA per tile; the tiles holding prefix query blocks (dense rows,
// several times longer) of all heads come first, then the video tiles head
// by head.
// The tile visits the union of its two query blocks' kept sets; a row whose
// block did not keep a visited key block masks it out and gets that block's
// pooled correction instead.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace sol {

constexpr int kTileM = 128;       // query rows per CTA (two 64-token blocks)
constexpr int kStageKeys = 64;    // keys per stage (one block)
constexpr int kRingStages = 2;    // depth of the K ring and of the V ring
constexpr int kMaxBlocks = 4096;  // largest M = N / 64 the router supports
constexpr int kMaskWords = kMaxBlocks / 32;
constexpr int kThreads = 192;
constexpr float kLog2Block = 6.0f;        // log2(64): the ln c_j bias in log2 units
constexpr float kRescaleSlack = 8.0f;     // keep a stale max while the new one is <= 2^8 larger
#ifndef SOL_ATTN_FMA_EXP_PAIRS
#define SOL_ATTN_FMA_EXP_PAIRS 2
#endif
// Of each 16 pairs of a 32-key half, this many take exp2 on the FMA pipe.
constexpr int kFmaExpPairs = SOL_ATTN_FMA_EXP_PAIRS;

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
  int skip_first_k_arrival;  // test hook: producer never loads stage 0
  int budget;                // > 0: keep this many top-scoring video blocks per query block
  bool correct;              // pooled correction of skipped blocks (else they are dropped)
  float out_scale;           // O is multiplied by this (the value scale of 8-bit V; 1 otherwise)
};

// kElem: bytes per element, 2 (bf16) or 1 (E4M3).  Tiles are stored in
// 128-byte column chunks (64 bf16 or 128 E4M3 values) with 128-byte swizzle.
template <int D, int kElem = 2>
struct SmemPlan {
  static constexpr int kBlockBytes = kStageKeys * D * kElem;  // one 64-key block of K (or V)
  static constexpr int kChunkBytes = kStageKeys * 128;        // its 128-byte column chunk (8 KB)
  static constexpr int kQChunkBytes = kTileM * 128;           // 128-byte column chunk of the Q tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileM * D * kElem;           // K ring
  static constexpr int kV = kK + kRingStages * kBlockBytes;  // V ring
  static constexpr int kMaskA = kV + kRingStages * kBlockBytes;
  static constexpr int kMaskB = kMaskA + kMaskWords * 4;
  static constexpr int kMaskU = kMaskB + kMaskWords * 4;
  static constexpr int kQbar = kMaskU + kMaskWords * 4;  // 2 x D floats
  static constexpr int kRed = kQbar + 2 * D * 4;         // 64 floats
  static constexpr int kHist = kRed + 64 * 4;            // 2 x 256 counters + 8 words (budget routing)
  static constexpr int kBars = kHist + (2 * 256 + 8) * 4;
  static constexpr int kNumBars = 4 * kRingStages + 2 + 6;
  static constexpr int kMisc = kBars + kNumBars * 8;     // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;           // room to align the base to 1 KB
  // The router's scores use the K and V rings before the first load.
  static constexpr int kScores = kK;
  static_assert(2 * kMaxBlocks * 4 <= 2 * kRingStages * kBlockBytes, "score scratch must fit in the rings");
};

// mbarriers: kfull[s], kempty[s], vfull[s], vempty[s], sfull[b], then singletons.
enum BarId {
  kBarKFull = 0,
  kBarKEmpty = kRingStages,
  kBarVFull = 2 * kRingStages,
  kBarVEmpty = 3 * kRingStages,
  kBarSFull = 4 * kRingStages,  // two S buffers
  kBarQ = 4 * kRingStages + 2,
  kBarPFull,
  kBarOReady,
  kBarOFull,
  kBarDrain,
};

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

// Video key blocks of the 32-block mask word starting at block `lo`.
__device__ __forceinline__ uint32_t video_bits(int lo, int M, int P) {
  if (lo >= M || lo + 32 <= P) return 0u;
  uint32_t v = lo < P ? (0xFFFFFFFFu << (P - lo)) : 0xFFFFFFFFu;
  if (M - lo < 32) v &= (1u << (M - lo)) - 1u;
  return v;
}

// The work of a tile, in order.  Exact stages: every block of the union of
// the two query blocks' kept sets, ascending.  Correction stages (unless
// the correction is off): pooled keys [64c, 64c + 64) holding at least one
// video block that either query block skipped.
struct Stage {
  int j;      // exact: key block; correction: pooled tile c
  bool corr;
};

// Number of stages StageIter yields for these masks, without walking them:
// popcount of the union plus the correction tiles that are needed.
__device__ __forceinline__ int count_stages(const uint32_t* mU, const uint32_t* mA, const uint32_t* mB,
                                            int M, int P, bool no_corr) {
  const int nw = (M + 31) >> 5;
  int n = 0;
  for (int w = 0; w < nw; ++w) n += __popc(mU[w]);
  if (no_corr) return n;
  for (int c = 0; c < ((M + 63) >> 6); ++c) {
    uint32_t any = 0u;
    for (int w = 2 * c; w < 2 * c + 2 && w < nw; ++w)
      any |= ((~mA[w]) | (~mB[w])) & video_bits(w * 32, M, P);
    n += any != 0u;
  }
  return n;
}

struct StageIter {
  int j = 0;
  int c = 0;
  __device__ __forceinline__ bool next(Stage& s, const uint32_t* mU, const uint32_t* mA,
                                       const uint32_t* mB, int M, int P, bool no_corr) {
    const int nw = (M + 31) >> 5;
    if (j < M) {
      const int j0 = next_bit(mU, j, nw);
      if (j0 >= 0) {
        s.j = j0;
        s.corr = false;
        j = j0 + 1;
        return true;
      }
      j = M;
    }
    if (no_corr) return false;
    const int nc = (M + 63) >> 6;
    while (c < nc) {
      const int cc = c++;
      const int w0 = cc * 2;
      uint32_t any = 0u;
      for (int w = w0; w < w0 + 2 && w < nw; ++w)
        any |= ((~mA[w]) | (~mB[w])) & video_bits(w * 32, M, P);
      if (any) {
        s.j = cc;
        s.corr = true;
        return true;
      }
    }
    return false;
  }
};

// CTA-wide (all kThreads threads) sum of two values / min-max of two pairs.
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ void cta_reduce2(float& a, float& b, float* red, int tid) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
  }
  __syncthreads();
  if ((tid & 31) == 0) {
    red[(tid >> 5) * 2] = a;
    red[(tid >> 5) * 2 + 1] = b;
  }
  __syncthreads();
  a = 0.f;
  b = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    a += red[2 * w];
    b += red[2 * w + 1];
  }
}

__device__ __forceinline__ void cta_reduce_minmax(float& mn_a, float& mx_a, float& mn_b, float& mx_b,
                                                  float* red, int tid) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn_a = fminf(mn_a, __shfl_xor_sync(0xFFFFFFFFu, mn_a, o));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xFFFFFFFFu, mx_a, o));
    mn_b = fminf(mn_b, __shfl_xor_sync(0xFFFFFFFFu, mn_b, o));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xFFFFFFFFu, mx_b, o));
  }
  __syncthreads();
  if ((tid & 31) == 0) {
    float* r = red + 2 * kWarps + (tid >> 5) * 4;
    r[0] = mn_a;
    r[1] = mx_a;
    r[2] = mn_b;
    r[3] = mx_b;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float* r = red + 2 * kWarps + w * 4;
    mn_a = fminf(mn_a, r[0]);
    mx_a = fmaxf(mx_a, r[1]);
    mn_b = fminf(mn_b, r[2]);
    mx_b = fmaxf(mx_b, r[3]);
  }
}

// Order-preserving map of an fp32 score to an unsigned key (larger score,
// larger key).
__device__ __forceinline__ uint32_t score_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Fixed-budget routing (draft stage): keep the `budget` highest scores of
// each video query block, ties at the cut going to the lower block index.
// The cut is found exactly by a 4-pass, 8-bit radix select over the score
// keys (shared-memory histograms, one warp picks each digit); a single warp
// then writes the keep words in block order, which settles ties.
template <int D, int kElem>
__device__ __forceinline__ void route_budget_masks(const AttnParams& p, const float* sc, uint8_t* smem,
                                                   int tid, bool videoA, bool videoB, bool hasB,
                                                   uint32_t* mA, uint32_t* mB) {
  using L = SmemPlan<D, kElem>;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L::kHist);  // [2][256]
  uint32_t* bc = hist + 512;                                      // broadcast words
  const int M = p.M, P = p.P, nv = M - P;
  const int nw = (M + 31) >> 5;
  const int kb = p.budget < nv ? p.budget : nv;
  uint32_t prefix[2] = {0u, 0u}, pmask = 0u;
  uint32_t need[2] = {static_cast<uint32_t>(kb), static_cast<uint32_t>(kb)};
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 512; i += kThreads) hist[i] = 0u;
    __syncthreads();
    for (int j = tid; j < nv; j += kThreads) {
      const uint32_t ua = score_key(sc[j]), ub = score_key(sc[kMaxBlocks + j]);
      if ((ua & pmask) == prefix[0]) atomicAdd(&hist[(ua >> shift) & 255u], 1u);
      if ((ub & pmask) == prefix[1]) atomicAdd(&hist[256 + ((ub >> shift) & 255u)], 1u);
    }
    __syncthreads();
    const int wq = tid >> 5, lane = tid & 31;
    if (wq < 2) {
      // Bins in descending digit order: lane l holds digits 255-8l .. 248-8l.
      const uint32_t* h = hist + 256 * wq;
      uint32_t loc[8], lsum = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        loc[i] = h[255 - 8 * lane - i];
        lsum += loc[i];
      }
      uint32_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t run = incl - lsum;  // keys in higher digits than this lane's bins
      const uint32_t nd = need[wq];
      int found = -1;
      uint32_t above = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (found < 0 && run < nd && nd <= run + loc[i]) {
          found = i;
          above = run;
        }
        run += loc[i];
      }
      const uint32_t who = __ballot_sync(0xFFFFFFFFu, found >= 0);
      if (who != 0u && lane == __ffs(who) - 1) {
        bc[2 * wq] = static_cast<uint32_t>(255 - 8 * lane - found);
        bc[2 * wq + 1] = above;
      }
    }
    __syncthreads();
    for (int q2 = 0; q2 < 2; ++q2) {
      prefix[q2] |= bc[2 * q2] << shift;
      need[q2] -= bc[2 * q2 + 1];
    }
    pmask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix[q] is now the key of the budget-th highest score; need[q] of the
  // keys equal to it are kept, lowest block first.
  if ((tid >> 5) == 0) {
    const int lane = tid & 31;
    uint32_t left[2] = {need[0], need[1]};
    for (int w = 0; w < nw; ++w) {
      const int j = w * 32 + lane;
      bool ka = j < M, kb2 = j < M;
      bool ea = false, eb = false;
      if (j >= P && j < M) {
        const uint32_t ua = score_key(sc[j - P]), ub = score_key(sc[kMaxBlocks + j - P]);
        if (videoA) {
          ka = ua > prefix[0];
          ea = ua == prefix[0];
        }
        if (videoB) {
          kb2 = ub > prefix[1];
          eb = ub == prefix[1];
        }
      }
      // ties at the cut: the first `left` of them in block order
      uint32_t tie = __ballot_sync(0xFFFFFFFFu, ea);
      const uint32_t rank_a = __popc(tie & ((1u << lane) - 1u));
      if (ea && rank_a < left[0]) ka = true;
      left[0] -= min(left[0], static_cast<uint32_t>(__popc(tie)));
      tie = __ballot_sync(0xFFFFFFFFu, eb);
      const uint32_t rank_b = __popc(tie & ((1u << lane) - 1u));
      if (eb && rank_b < left[1]) kb2 = true;
      left[1] -= min(left[1], static_cast<uint32_t>(__popc(tie)));
      const uint32_t wa = __ballot_sync(0xFFFFFFFFu, ka);
      const uint32_t wb = __ballot_sync(0xFFFFFFFFu, kb2);
      if (lane == 0) {
        mA[w] = wa;
        mB[w] = hasB ? wb : wa;
      }
    }
  }
}

// Router: pooled scores of query blocks iA, iB against every video key
// block, population mean/std, threshold, keep bits.  Runs on all the CTA's
// threads before the mainloop; scores live in the (not yet used) K/V rings.
template <int D, int kElem>
__device__ __forceinline__ void route_tile(const AttnParams& p, int bh, int iA, int iB, bool hasB,
                                           uint8_t* smem, int tid, float pre_a, float pre_b) {
  using L = SmemPlan<D, kElem>;
  uint32_t* mA = reinterpret_cast<uint32_t*>(smem + L::kMaskA);
  uint32_t* mB = reinterpret_cast<uint32_t*>(smem + L::kMaskB);
  float* sq = reinterpret_cast<float*>(smem + L::kQbar);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* sc = reinterpret_cast<float*>(smem + L::kScores);  // [2][kMaxBlocks]
  const int M = p.M, P = p.P, nv = M - P;
  const int nw = (M + 31) >> 5;
  const bool videoA = iA >= P, videoB = hasB && iB >= P;

  if ((videoA || videoB) && nv > 0) {
    // The pooled queries were loaded at kernel entry (thread d holds dim d).
    static_assert(D <= kThreads, "one pooled-query dimension per thread");
    if (tid < D) {
      sq[tid] = pre_a;
      sq[D + tid] = pre_b;
    }
    __syncthreads();
    // Scores, 32 key blocks per warp step: lane l holds dims [D/32 * l, +D/32)
    // of every row, so each row is one coalesced load of the warp; the 32
    // partial dot products per lane are then reduced across lanes by a
    // butterfly that leaves row (base + l)'s score in lane l.
    {
      constexpr int kDpl = D / 32;  // dims per lane: 4 (D = 128) or 2 (D = 64)
      const int lane = tid & 31, wq = tid >> 5;
      float qa[kDpl], qb[kDpl];
#pragma unroll
      for (int d = 0; d < kDpl; ++d) {
        qa[d] = sq[lane * kDpl + d];
        qb[d] = sq[D + lane * kDpl + d];
      }
      const float* kb = p.kbar + static_cast<size_t>(bh) * M * D + lane * kDpl;
      for (int base = P + wq * 32; base < M; base += 32 * kWarps) {
        float pa[32], pb[32];
#pragma unroll
        for (int rr = 0; rr < 32; ++rr) {
          const int j = base + rr;
          float kv[kDpl];
          if (j < M) {
            if constexpr (kDpl == 4) {
              const float4 x = __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D));
              kv[0] = x.x; kv[1] = x.y; kv[2] = x.z; kv[3] = x.w;
            } else {
              const float2 x = __ldg(reinterpret_cast<const float2*>(kb + static_cast<size_t>(j) * D));
              kv[0] = x.x; kv[1] = x.y;
            }
          } else {
#pragma unroll
            for (int d = 0; d < kDpl; ++d) kv[d] = 0.f;
          }
          float da = 0.f, db = 0.f;
#pragma unroll
          for (int d = 0; d < kDpl; ++d) {
            da = fmaf(qa[d], kv[d], da);
            db = fmaf(qb[d], kv[d], db);
          }
          pa[rr] = da;
          pb[rr] = db;
        }
#pragma unroll
        for (int lvl = 16; lvl >= 1; lvl >>= 1) {
          const bool upper = (lane & lvl) != 0;
#pragma unroll
          for (int i = 0; i < lvl; ++i) {
            const float sa = upper ? pa[i] : pa[i + lvl];
            const float ka = upper ? pa[i + lvl] : pa[i];
            const float sb = upper ? pb[i] : pb[i + lvl];
            const float kb2 = upper ? pb[i + lvl] : pb[i];
            pa[i] = ka + __shfl_xor_sync(0xFFFFFFFFu, sa, lvl);
            pb[i] = kb2 + __shfl_xor_sync(0xFFFFFFFFu, sb, lvl);
          }
        }
        const int j = base + lane;
        if (j < M) {
          sc[j - P] = pa[0] * p.scale;
          sc[kMaxBlocks + j - P] = pb[0] * p.scale;
        }
      }
    }
    __syncthreads();
    if (p.budget > 0) {
      route_budget_masks<D, kElem>(p, sc, smem, tid, videoA, videoB, hasB, mA, mB);
      return;
    }
    // Pass 1: mean (and exact-equality check through min/max).
    float sa = 0.f, sb = 0.f;
    float mna = INFINITY, mxa = -INFINITY, mnb = INFINITY, mxb = -INFINITY;
    for (int j = tid; j < nv; j += kThreads) {
      const float a = sc[j], b = sc[kMaxBlocks + j];
      sa += a; sb += b;
      mna = fminf(mna, a); mxa = fmaxf(mxa, a);
      mnb = fminf(mnb, b); mxb = fmaxf(mxb, b);
    }
    cta_reduce2(sa, sb, red, tid);
    cta_reduce_minmax(mna, mxa, mnb, mxb, red, tid);
    const float mua = sa / nv, mub = sb / nv;
    // Pass 2: population variance about the mean.
    float va = 0.f, vb = 0.f;
    for (int j = tid; j < nv; j += kThreads) {
      const float a = sc[j] - mua, b = sc[kMaxBlocks + j] - mub;
      va = fmaf(a, a, va);
      vb = fmaf(b, b, vb);
    }
    __syncthreads();  // everyone has read red[] of the previous reduction
    cta_reduce2(va, vb, red, tid);
    const float sda = (mna == mxa) ? 0.f : sqrtf(va / nv);
    const float sdb = (mnb == mxb) ? 0.f : sqrtf(vb / nv);
    const bool allA = (p.tau == -INFINITY) || sda == 0.f;
    const bool allB = (p.tau == -INFINITY) || sdb == 0.f;
    const float thrA = mua + p.tau * sda;
    const float thrB = mub + p.tau * sdb;
    // Keep bits, one 32-block word per warp iteration.
    const int lane = tid & 31, wq = tid >> 5;
    for (int w = wq; w < nw; w += kWarps) {
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
    for (int w = tid; w < nw; w += kThreads) {
      const int lo = w * 32;
      const uint32_t full = (M - lo >= 32) ? 0xFFFFFFFFu : ((1u << (M - lo)) - 1u);
      mA[w] = full;
      mB[w] = full;
    }
  }
}

template <int D, bool kDense, bool kFp8 = false>
__global__ void __launch_bounds__(kThreads, 2)
    sol_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKb,
                        const __grid_constant__ CUtensorMap tmVb, const AttnParams p) {
  // kFp8: E4M3 Q, K, V and pooled K/V, tcgen05.mma kind::f8f6f4 (32 values of K
  // per instruction), P stored to TMEM as E4M3, four per column.
  constexpr int kElem = kFp8 ? 1 : 2;
  using L = SmemPlan<D, kElem>;
  constexpr int kChunks = D * kElem / 128;
  constexpr int kChunkElems = 128 / kElem;   // values per 128-byte chunk row
  constexpr int kMmaK = 32 / kElem;          // K of one MMA instruction
  static_assert(!kFp8 || D == 128, "the 8-bit path is built for D = 128");
  constexpr uint32_t kTmemCols = 256;
  constexpr uint32_t kColO = 128;  // S buffer b at columns [64 b, 64 b + 64)

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
  const int M = p.M, P = p.P;
  // Launch order: a tile holding a prefix query block attends to every key
  // block and runs several times longer than a video tile, so the prefix
  // tiles of all heads come first and the video tiles follow, head by head.
  // The long tiles then never form the tail of the grid.
  int bh = static_cast<int>(blockIdx.x) / p.tiles_per_head;
  int qt = static_cast<int>(blockIdx.x) % p.tiles_per_head;
  if constexpr (!kDense) {
    const int T = p.tiles_per_head;
    const int PT = min(T, (P + 1) / 2);  // tiles holding a prefix query block
    const int idx = static_cast<int>(blockIdx.x), nlong = p.B * p.H * PT;
    if (idx < nlong) {
      bh = idx / PT;
      qt = idx % PT;
    } else {
      bh = (idx - nlong) / (T - PT);
      qt = PT + (idx - nlong) % (T - PT);
    }
  }
  const int iA = 2 * qt, iB = 2 * qt + 1;
  const bool hasB = iB < M;
  const int nw = (M + 31) >> 5;
  const bool no_corr = kDense || !p.correct;
  int* err = &g_sol_attn_error;

  // The router's pooled queries are loaded first thing, so their global
  // latency overlaps the barrier, TMEM and Q-tile setup below.
  float pre_qa = 0.f, pre_qb = 0.f;
  if (!kDense && tid < D && p.qbar != nullptr && ((iA >= P) || (hasB && iB >= P)) && M > P) {
    pre_qa = __ldg(p.qbar + (static_cast<size_t>(bh) * M + iA) * D + tid);
    pre_qb = __ldg(p.qbar + (static_cast<size_t>(bh) * M + (hasB ? iB : iA)) * D + tid);
  }
  if (tid == 0) {
    for (int i = 0; i < kRingStages; ++i) {
      mbar_init(&bars[kBarKFull + i], 1);
      mbar_init(&bars[kBarKEmpty + i], 1);
      mbar_init(&bars[kBarVFull + i], 1);
      mbar_init(&bars[kBarVEmpty + i], 1);
    }
    mbar_init(&bars[kBarSFull + 0], 1);
    mbar_init(&bars[kBarSFull + 1], 1);
    mbar_init(&bars[kBarQ], 1);
    mbar_init(&bars[kBarPFull], 128);
    mbar_init(&bars[kBarOReady], 1);
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
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    const size_t row0 = static_cast<size_t>(bh) * p.N + static_cast<size_t>(qt) * kTileM;
    mbar_arrive_expect_tx(&bars[kBarQ], kTileM * D * kElem);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        tma_load_2d(sQ + c * L::kQChunkBytes + h * 64 * 128, &tmQ, &bars[kBarQ], c * kChunkElems,
                    static_cast<int>(row0 + h * 64));
  }

  // Routing on all threads (the producer has already issued the Q load), or
  // the all-kept mask of the dense kernel.
  if (kDense) {
    for (int w = tid; w < nw; w += kThreads) {
      const int lo = w * 32;
      const uint32_t fullw = (M - lo >= 32) ? 0xFFFFFFFFu : ((1u << (M - lo)) - 1u);
      mA[w] = fullw;
      mB[w] = fullw;
    }
  } else {
    route_tile<D, kElem>(p, bh, iA, iB, hasB, smem, tid, pre_qa, pre_qb);
  }
  __syncthreads();
  for (int w = tid; w < nw; w += kThreads) mU[w] = mA[w] | mB[w];
  if (!kDense && (p.debug_mask != nullptr || p.kept_pairs != nullptr || p.exact_pairs != nullptr)) {
    unsigned long long kept = 0, uni = 0;
    for (int w = tid; w < nw; w += kThreads) {
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
  fence_proxy_async_smem();  // scores were written to the rings by generic stores
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
      uint32_t k_issued[kRingStages] = {}, v_issued[kRingStages] = {};
      while (ok && it.next(s, mU, mA, mB, M, P, no_corr)) {
        const int slot = n % kRingStages;
        const uint32_t use_parity = ((n / kRingStages) - 1) & 1;
        const int row = static_cast<int>(s.corr ? prow_head + static_cast<size_t>(s.j) * 64
                                                : krow_head + static_cast<size_t>(s.j) * 64);
        if (n >= kRingStages)
          ok = mbar_wait(&bars[kBarKEmpty + slot], use_parity, abort_flag, err, 1, p.timeout_ns);
        if (!ok) break;
        if (!(p.skip_first_k_arrival && n == 0)) {
          mbar_arrive_expect_tx(&bars[kBarKFull + slot], L::kBlockBytes);
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(sK + slot * L::kBlockBytes + c * L::kChunkBytes, s.corr ? &tmKb : &tmK,
                        &bars[kBarKFull + slot], c * kChunkElems, row);
          ++k_issued[slot];
        }
        if (n >= kRingStages)
          ok = mbar_wait(&bars[kBarVEmpty + slot], use_parity, abort_flag, err, 2, p.timeout_ns);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars[kBarVFull + slot], L::kBlockBytes);
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(sV + slot * L::kBlockBytes + c * L::kChunkBytes, s.corr ? &tmVb : &tmV,
                      &bars[kBarVFull + slot], c * kChunkElems, row);
        ++v_issued[slot];
        ++n;
      }
      if (!ok || *abort_flag) {
        // Let the loads already issued land before the CTA's shared memory is
        // released: the k-th load into a ring slot completes phase k - 1 of
        // its full barrier (bounded waits that ignore the abort flag).
        for (int i = 0; i < kRingStages; ++i) {
          if (k_issued[i] > 0) mbar_wait_drain(&bars[kBarKFull + i], (k_issued[i] - 1) & 1, p.timeout_ns);
          if (v_issued[i] > 0) mbar_wait_drain(&bars[kBarVFull + i], (v_issued[i] - 1) & 1, p.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors are built once.  A ring slot or k-step only moves the
      // start-address field (shared address >> 4, below 2^14, so adding an
      // offset never carries): one add per MMA on the issue path, which
      // shares its SMSP with softmax warps.
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t vdesc = sdesc_sw128(smem_u32(sV), L::kChunkBytes, 1024);
      const uint32_t idesc_qk = kFp8 ? idesc_e4m3_f32(kTileM, kStageKeys, false)
                                     : idesc_bf16_f32(kTileM, kStageKeys, false);
      const uint32_t idesc_pv = kFp8 ? idesc_e4m3_f32(kTileM, D, true) : idesc_bf16_f32(kTileM, D, true);
      const int total = count_stages(mU, mA, mB, M, P, no_corr);
      bool ok = mbar_wait(&bars[kBarQ], 0, abort_flag, err, 3, p.timeout_ns);
      // S(n) = Q K(n)^T into S buffer n % 2; A = Q (K-major SW128), B = K.
      auto issue_s = [&](int n) -> bool {
        const int slot = n % kRingStages;
        if (!mbar_wait(&bars[kBarKFull + slot], (n / kRingStages) & 1, abort_flag, err, 4, p.timeout_ns))
          return false;
        tc_fence_after();
        const uint64_t kd = kdesc + static_cast<uint32_t>((slot * L::kBlockBytes) >> 4);
        const uint32_t dcol = tmem + 64u * (n & 1);
#pragma unroll
        for (int kk = 0; kk < D / kMmaK; ++kk) {
          // 32 bytes of K per instruction: four steps per 128-byte chunk.
          constexpr int kQStep = L::kQChunkBytes >> 4, kKStep = L::kChunkBytes >> 4;
          const uint64_t ad = qdesc + static_cast<uint32_t>((kk >> 2) * kQStep + (kk & 3) * 2);
          const uint64_t bd = kd + static_cast<uint32_t>((kk >> 2) * kKStep + (kk & 3) * 2);
          if constexpr (kFp8)
            mma_e4m3_ss(dcol, ad, bd, idesc_qk, kk > 0);
          else
            mma_bf16_ss(dcol, ad, bd, idesc_qk, kk > 0);
        }
        mma_commit(&bars[kBarSFull + (n & 1)]);
        mma_commit(&bars[kBarKEmpty + slot]);
        return true;
      };
      if (ok && total > 0) ok = issue_s(0);
      if (ok && total > 1) ok = issue_s(1);
      for (int n = 0; ok && n < total; ++n) {
        const int slot = n % kRingStages;
        ok = mbar_wait(&bars[kBarPFull], n & 1, abort_flag, err, 5, p.timeout_ns);
        if (ok) ok = mbar_wait(&bars[kBarVFull + slot], (n / kRingStages) & 1, abort_flag, err, 6, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        // O += P V: A = P from S buffer n % 2 (TMEM), B = V (MN-major).
        const uint32_t pcol = tmem + 64u * (n & 1);
        const uint64_t vd = vdesc + static_cast<uint32_t>((slot * L::kBlockBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kStageKeys / kMmaK; ++kk) {
          // kMmaK keys per instruction: 32 bytes of P (8 TMEM columns) and
          // kMmaK 128-byte rows of V.
          const uint64_t bd = vd + static_cast<uint32_t>(kk * ((kMmaK * 128) >> 4));
          if constexpr (kFp8)
            mma_e4m3_ts(tmem + kColO, pcol + kk * 8, bd, idesc_pv, (n > 0 || kk > 0) ? 1u : 0u);
          else
            mma_bf16_ts(tmem + kColO, pcol + kk * 8, bd, idesc_pv, (n > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kBarVEmpty + slot]);
        mma_commit(&bars[kBarOReady]);
        // The next S into this buffer runs after this PV (tcgen05.mma from one
        // thread executes in issue order), so P is read before it is overwritten.
        if (n + 2 < total) ok = issue_s(n + 2);
      }
      mma_commit(&bars[kBarOFull]);
      mma_commit(&bars[kBarDrain]);
      // Drain: the CTA must not free TMEM while MMAs are still running.
      mbar_wait_drain(&bars[kBarDrain], 0, 2000000000ull);
      // A Q tile whose wait gave up must still land before shared memory is released.
      if (!ok) mbar_wait_drain(&bars[kBarQ], 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int sp = warp & 3;
    const int r = sp * 32 + lane;
    const uint32_t* rowmask = r < 64 ? mA : mB;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sp * 32) << 16);
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    float m = -INFINITY, l = 0.f;
    StageIter it;
    Stage s;
    int n = 0;
    bool ok = true;
    while (it.next(s, mU, mA, mB, M, P, no_corr)) {
      const uint32_t scol = lane_addr + 64u * (n & 1);
      ok = mbar_wait(&bars[kBarSFull + (n & 1)], (n >> 1) & 1, abort_flag, err, 7, p.timeout_ns);
      if (!ok) break;
      tc_fence_after();
      // Which of the 64 columns this row uses (warp-uniform: one query block per warp).
      uint32_t use0, use1;
      if (!s.corr) {
        use0 = use1 = mask_bit(rowmask, s.j) ? 0xFFFFFFFFu : 0u;
      } else {
        const int lo = s.j * 64;
        const uint32_t v0 = video_bits(lo, M, P), v1 = video_bits(lo + 32, M, P);
        use0 = v0 ? (~rowmask[lo >> 5] & v0) : 0u;
        use1 = v1 ? (~rowmask[(lo >> 5) + 1] & v1) : 0u;
      }
      uint32_t pk0[16], pk1[16];
      float ea0 = 0.f, ea1 = 0.f, eb0 = 0.f, eb1 = 0.f;  // E4M3 path: the even pair of a column
      float alpha = 1.0f;
      bool warp_need = false;
      if (__any_sync(0xFFFFFFFFu, (use0 | use1) != 0u)) {
        uint32_t sv0[32], sv1[32];
        tmem_ld32(scol + 0, sv0);
        tmem_ld32(scol + 32, sv1);
        tmem_ld_wait(sv0);
        tmem_ld_wait(sv1);
        // Row max on raw scores (scale > 0), independent chains.
        float tmax = -INFINITY;
        if (!s.corr) {
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            m0 = max3f(m0, __uint_as_float(sv0[c]), __uint_as_float(sv0[c + 1]));
            m1 = max3f(m1, __uint_as_float(sv0[c + 2]), __uint_as_float(sv0[c + 3]));
            m2 = max3f(m2, __uint_as_float(sv1[c]), __uint_as_float(sv1[c + 1]));
            m3 = max3f(m3, __uint_as_float(sv1[c + 2]), __uint_as_float(sv1[c + 3]));
          }
          tmax = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * p.scale_log2;
        } else {
          float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            m0 = fmaxf(m0, ((use0 >> c) & 1u) ? __uint_as_float(sv0[c]) : -INFINITY);
            m1 = fmaxf(m1, ((use1 >> c) & 1u) ? __uint_as_float(sv1[c]) : -INFINITY);
          }
          const float mraw = fmaxf(m0, m1);
          if (mraw != -INFINITY) tmax = fmaf(mraw, p.scale_log2, kLog2Block);
        }
        // Online softmax with a stale max: O is rescaled only when the running
        // max grows by more than 2^8; m, l and O always share one reference.
        const bool need = (m != -INFINITY) && (tmax > m + kRescaleSlack);
        warp_need = __any_sync(0xFFFFFFFFu, need);
        alpha = need ? fast_exp2(m - tmax) : 1.0f;
        if (need || (m == -INFINITY && tmax > m)) m = tmax;
        const float mref = (m == -INFINITY) ? 0.f : m;
        const float bias = (s.corr ? kLog2Block : 0.f) - mref;
        const uint64_t bias2 = f2_pack(bias, bias);
        uint64_t acc0 = 0ull, acc1 = 0ull, acc2 = 0ull, acc3 = 0ull;
        if (!s.corr) {
          // Every column used: no per-element masking.
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t xa = f2_fma(f2_pack(__uint_as_float(sv0[2 * c]), __uint_as_float(sv0[2 * c + 1])),
                                       scale2, bias2);
            const uint64_t xb = f2_fma(f2_pack(__uint_as_float(sv1[2 * c]), __uint_as_float(sv1[2 * c + 1])),
                                       scale2, bias2);
            float a0, a1, b0, b1;
            if (c >= 16 - kFmaExpPairs) {
              exp2_fma_pair(xa, a0, a1);
              exp2_fma_pair(xb, b0, b1);
            } else {
              f2_unpack(xa, a0, a1);
              f2_unpack(xb, b0, b1);
              a0 = fast_exp2(a0);
              a1 = fast_exp2(a1);
              b0 = fast_exp2(b0);
              b1 = fast_exp2(b1);
            }
            const uint64_t pa = f2_pack(a0, a1), pb = f2_pack(b0, b1);
            if (c & 1) {
              acc1 = f2_add(acc1, pa);
              acc3 = f2_add(acc3, pb);
            } else {
              acc0 = f2_add(acc0, pa);
              acc2 = f2_add(acc2, pb);
            }
            if constexpr (kFp8) {
              if (c & 1) {
                pk0[c >> 1] = pack_e4m3x4(ea0, ea1, a0, a1);
                pk1[c >> 1] = pack_e4m3x4(eb0, eb1, b0, b1);
              } else {
                ea0 = a0; ea1 = a1; eb0 = b0; eb1 = b1;
              }
            } else {
              pk0[c] = pack_bf16x2(a0, a1);
              pk1[c] = pack_bf16x2(b0, b1);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t xa = f2_fma(f2_pack(__uint_as_float(sv0[2 * c]), __uint_as_float(sv0[2 * c + 1])),
                                       scale2, bias2);
            const uint64_t xb = f2_fma(f2_pack(__uint_as_float(sv1[2 * c]), __uint_as_float(sv1[2 * c + 1])),
                                       scale2, bias2);
            float a0, a1, b0, b1;
            f2_unpack(xa, a0, a1);
            f2_unpack(xb, b0, b1);
            a0 = ((use0 >> (2 * c)) & 1u) ? fast_exp2(a0) : 0.f;
            a1 = ((use0 >> (2 * c + 1)) & 1u) ? fast_exp2(a1) : 0.f;
            b0 = ((use1 >> (2 * c)) & 1u) ? fast_exp2(b0) : 0.f;
            b1 = ((use1 >> (2 * c + 1)) & 1u) ? fast_exp2(b1) : 0.f;
            const uint64_t pa = f2_pack(a0, a1), pb = f2_pack(b0, b1);
            if (c & 1) {
              acc1 = f2_add(acc1, pa);
              acc3 = f2_add(acc3, pb);
            } else {
              acc0 = f2_add(acc0, pa);
              acc2 = f2_add(acc2, pb);
            }
            if constexpr (kFp8) {
              if (c & 1) {
                pk0[c >> 1] = pack_e4m3x4(ea0, ea1, a0, a1);
                pk1[c >> 1] = pack_e4m3x4(eb0, eb1, b0, b1);
              } else {
                ea0 = a0; ea1 = a1; eb0 = b0; eb1 = b1;
              }
            } else {
              pk0[c] = pack_bf16x2(a0, a1);
              pk1[c] = pack_bf16x2(b0, b1);
            }
          }
        }
        const uint64_t a = f2_add(f2_add(acc0, acc1), f2_add(acc2, acc3));
        float s0, s1;
        f2_unpack(a, s0, s1);
        l = fmaf(l, alpha, s0 + s1);
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          pk0[c] = 0u;
          pk1[c] = 0u;
        }
      }
      if constexpr (kFp8) {
        // 64 keys of E4M3 P: columns 0-7 from the first 32 keys, 8-15 from the rest.
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pk[i] = pk0[i];
          pk[8 + i] = pk1[i];
        }
        tmem_st16(scol + 0, pk);
      } else {
        tmem_st16(scol + 0, pk0);
        tmem_st16(scol + 16, pk1);
      }
      // Every stage n >= 1 waits for PV(n-1) (the n-th commit on OReady).
      // Waiting each time keeps the parity unambiguous: PV(n-2) is known to
      // be done, so only phase n-1 can be pending.  The wait sits after this
      // stage's math, by when PV(n-1) has normally finished.
      if (n > 0) {
        ok = mbar_wait(&bars[kBarOReady], (n - 1) & 1, abort_flag, err, 9, p.timeout_ns);
        if (!ok) break;
      }
      // O *= alpha, with no PV in flight: PV(n-1) is done and PV(n) waits
      // for the arrival below.  tcgen05.ld/st are warp-collective, so the
      // pass runs when any row of the warp needs it (alpha = 1 for the others).
      if (warp_need) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + c0, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(lane_addr + kColO + c0, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[kBarPFull]);
      ++n;
    }
    // Epilogue: out = O / l.
    if (ok) ok = mbar_wait(&bars[kBarOFull], 0, abort_flag, err, 8, p.timeout_ns);
    if (ok) {
      tc_fence_after();
      const float inv_l = l > 0.f ? p.out_scale / l : 0.f;
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
