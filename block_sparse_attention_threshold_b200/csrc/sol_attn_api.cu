// Host side of the C ABI declared in include/sol_attn.h: argument checks,
// workspace, TMA descriptors, kernel launches and the host-buffer pipeline.
// No torch.  No host syncs, except in sol_attn_device_status and in
// sol_attn_forward_host: on its error path (when the stream ordering of its
// tail cannot be enqueued, it drains its own streams before freeing the
// scratch), and when `out` is pageable host memory (the runtime then makes
// each device-to-host copy return only once it has finished).
#include "sol_attn.h"

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "attn_kernel.cuh"
#include "pool_kernel.cuh"
#include "prep_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceCache {
  std::once_flag once;
  int status = SOL_ATTN_OK;  // SOL_ATTN_OK or SOL_ATTN_ERR_ARCH / _CUDA
};
DeviceCache g_dev[kMaxDevices];

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SOL_ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SOL_ATTN_ERR_UNSUPPORTED;
  DeviceCache& c = g_dev[dev];
  std::call_once(c.once, [&] {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      c.status = SOL_ATTN_ERR_CUDA;
      return;
    }
    if (major != 10 || minor != 0) {
      c.status = SOL_ATTN_ERR_ARCH;
      return;
    }
    // Opt the attention kernels into their shared-memory footprint.
    bool ok = true;
    ok &= cudaFuncSetAttribute(sol::sol_attn_fwd_kernel<128, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sol::SmemPlan<128>::kAlloc) == cudaSuccess;
    ok &= cudaFuncSetAttribute(sol::sol_attn_fwd_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sol::SmemPlan<128>::kAlloc) == cudaSuccess;
    ok &= cudaFuncSetAttribute(sol::sol_attn_fwd_kernel<64, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sol::SmemPlan<64>::kAlloc) == cudaSuccess;
    ok &= cudaFuncSetAttribute(sol::sol_attn_fwd_kernel<64, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sol::SmemPlan<64>::kAlloc) == cudaSuccess;
    ok &= cudaFuncSetAttribute(sol::sol_attn_fwd_kernel<128, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sol::SmemPlan<128, 1>::kAlloc) == cudaSuccess;
    c.status = ok ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
  });
  return c.status;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D view [rows, D] of a bf16 array, 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2D view [rows, D] of an 8-bit array (E4M3 bytes), 64-row x 128-byte boxes,
// 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Shape checks shared by every entry point.  Returns SOL_ATTN_OK, an error,
// or -1 for an empty problem (nothing to do).
int check_shape(int B, int H, int N, int D) {
  if (B < 0 || H < 0 || N < 0) return SOL_ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SOL_ATTN_ERR_UNSUPPORTED;
  if (N % SOL_ATTN_BLOCK != 0) return SOL_ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return -1;
  if (N / SOL_ATTN_BLOCK > sol::kMaxBlocks) return SOL_ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N > INT_MAX) return SOL_ATTN_ERR_UNSUPPORTED;
  return SOL_ATTN_OK;
}

int check_io(const void* q, const void* k, const void* v, const void* out) {
  if (!q || !k || !v || !out) return SOL_ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return SOL_ATTN_ERR_INVALID_ARG;
  return SOL_ATTN_OK;
}

int check_opts(const sol_attn_opts* o) {
  if (o == nullptr) return SOL_ATTN_OK;
  if (!(std::isfinite(o->softmax_scale)) || o->softmax_scale < 0.f) return SOL_ATTN_ERR_INVALID_ARG;
  if (o->budget_blocks < 0) return SOL_ATTN_ERR_INVALID_ARG;
  return SOL_ATTN_OK;
}

struct Workspace {
  float* qbar;
  float* kbar;
  __nv_bfloat16* kbar_bf16;
  __nv_bfloat16* vbar_bf16;
};

Workspace split_workspace(const void* ws, int B, int H, int N, int D) {
  size_t off[4];
  sol_attn_workspace_bytes(B, H, N, D, off);
  auto* b = static_cast<uint8_t*>(const_cast<void*>(ws));
  return Workspace{reinterpret_cast<float*>(b + off[0]), reinterpret_cast<float*>(b + off[1]),
                   reinterpret_cast<__nv_bfloat16*>(b + off[2]),
                   reinterpret_cast<__nv_bfloat16*>(b + off[3])};
}

int launch_pool(const void* q, const void* k, const void* v, const Workspace& w, int B, int H,
                int N, int D, cudaStream_t s) {
  const unsigned nblk = static_cast<unsigned>(static_cast<long long>(B) * H * (N / SOL_ATTN_BLOCK));
  sol::PoolOut o{w.qbar, w.kbar, w.kbar_bf16, w.vbar_bf16};
  dim3 grid(nblk, 3);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  if (D == 128)
    sol::pool_kernel<128><<<grid, 128, 0, s>>>(qb, kb, vb, o);
  else
    sol::pool_kernel<64><<<grid, 128, 0, s>>>(qb, kb, vb, o);
  return cudaGetLastError() == cudaSuccess ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

int launch_attend(const void* q, const void* k, const void* v, void* out, const Workspace* w,
                  int B, int H, int N, int D, float tau, int prefix_len, const sol_attn_opts* o,
                  bool dense, cudaStream_t s) {
  const int M = N / SOL_ATTN_BLOCK;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N;
  const uint64_t prows = static_cast<uint64_t>(B) * H * M;
  CUtensorMap mq, mk, mv, mkb, mvb;
  if (!make_map(&mq, q, rows, D) || !make_map(&mk, k, rows, D) || !make_map(&mv, v, rows, D))
    return SOL_ATTN_ERR_CUDA;
  if (w != nullptr) {
    if (!make_map(&mkb, w->kbar_bf16, prows, D) || !make_map(&mvb, w->vbar_bf16, prows, D))
      return SOL_ATTN_ERR_CUDA;
  } else {
    mkb = mk;
    mvb = mv;
  }
  sol::AttnParams p{};
  p.B = B;
  p.H = H;
  p.N = N;
  p.M = M;
  p.P = prefix_len / SOL_ATTN_BLOCK;
  p.tiles_per_head = (M + 1) / 2;
  p.tau = tau;
  const float scale = (o != nullptr && o->softmax_scale > 0.f) ? o->softmax_scale
                                                               : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.qbar = w ? w->qbar : nullptr;
  p.kbar = w ? w->kbar : nullptr;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.debug_mask = o ? o->debug_mask : nullptr;
  p.kept_pairs = o ? o->kept_pairs : nullptr;
  p.exact_pairs = o ? o->exact_pairs : nullptr;
  const unsigned tms = (o != nullptr && o->timeout_ms > 0) ? o->timeout_ms : 1000u;
  p.timeout_ns = static_cast<uint64_t>(tms) * 1000000ull;
  p.skip_first_k_arrival = o ? o->test_skip_first_k_load : 0;
  p.budget = o ? o->budget_blocks : 0;
  p.correct = !(o != nullptr && o->skip_correction != 0);
  p.out_scale = 1.0f;

  const long long tiles = static_cast<long long>(B) * H * p.tiles_per_head;
  dim3 grid(static_cast<unsigned>(tiles));
  if (D == 128) {
    const int smem = sol::SmemPlan<128>::kAlloc;
    if (dense)
      sol::sol_attn_fwd_kernel<128, true><<<grid, sol::kThreads, smem, s>>>(mq, mk, mv, mkb, mvb, p);
    else
      sol::sol_attn_fwd_kernel<128, false><<<grid, sol::kThreads, smem, s>>>(mq, mk, mv, mkb, mvb, p);
  } else {
    const int smem = sol::SmemPlan<64>::kAlloc;
    if (dense)
      sol::sol_attn_fwd_kernel<64, true><<<grid, sol::kThreads, smem, s>>>(mq, mk, mv, mkb, mvb, p);
    else
      sol::sol_attn_fwd_kernel<64, false><<<grid, sol::kThreads, smem, s>>>(mq, mk, mv, mkb, mvb, p);
  }
  return cudaGetLastError() == cudaSuccess ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

int check_route_args(int block, float tau, int prefix_len, int N) {
  if (block != SOL_ATTN_BLOCK) return SOL_ATTN_ERR_UNSUPPORTED;
  if (std::isnan(tau)) return SOL_ATTN_ERR_INVALID_ARG;
  if (prefix_len < 0 || prefix_len > N || prefix_len % SOL_ATTN_BLOCK != 0)
    return SOL_ATTN_ERR_INVALID_ARG;
  return SOL_ATTN_OK;
}

}  // namespace

extern "C" {

size_t sol_attn_workspace_bytes(int B, int H, int N, int D, size_t* offsets) {
  const int sc = check_shape(B, H, N, D);
  if (sc != SOL_ATTN_OK) {
    if (offsets) std::memset(offsets, 0, 4 * sizeof(size_t));
    return 0;
  }
  const size_t rows = static_cast<size_t>(B) * H * (N / SOL_ATTN_BLOCK);
  const size_t f32 = round256(rows * D * 4), b16 = round256(rows * D * 2);
  if (offsets) {
    offsets[0] = 0;
    offsets[1] = f32;
    offsets[2] = 2 * f32;
    offsets[3] = 2 * f32 + b16;
  }
  return 2 * f32 + 2 * b16;
}

int sol_attn_pool(const void* q, const void* k, const void* v, void* workspace, int B, int H,
                  int N, int D, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return SOL_ATTN_OK;
  if (st != SOL_ATTN_OK) return st;
  if (!q || !k || !v || !workspace || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  return launch_pool(q, k, v, split_workspace(workspace, B, H, N, D), B, H, N, D,
                     static_cast<cudaStream_t>(stream));
}

int sol_attn_attend(const void* q, const void* k, const void* v, void* out, const void* workspace,
                    int B, int H, int N, int D, int block, float tau, int prefix_len,
                    const sol_attn_opts* opts, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_opts(opts)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  const Workspace w = split_workspace(workspace, B, H, N, D);
  return launch_attend(q, k, v, out, &w, B, H, N, D, tau, prefix_len, opts, false,
                       static_cast<cudaStream_t>(stream));
}

int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out, int B, int H,
                        int N, int D, int block, float tau, int prefix_len,
                        const sol_attn_opts* opts, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if ((st = check_opts(opts)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = sol_attn_workspace_bytes(B, H, N, D, nullptr);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, s) != cudaSuccess) return SOL_ATTN_ERR_CUDA;
  const Workspace w = split_workspace(ws, B, H, N, D);
  st = launch_pool(q, k, v, w, B, H, N, D, s);
  if (st == SOL_ATTN_OK) st = launch_attend(q, k, v, out, &w, B, H, N, D, tau, prefix_len, opts, false, s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && st == SOL_ATTN_OK) st = SOL_ATTN_ERR_CUDA;
  return st;
}

int sol_attn_forward(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                     int D, int block, float tau, int prefix_len, void* stream) {
  return sol_attn_forward_ex(q, k, v, out, B, H, N, D, block, tau, prefix_len, nullptr, stream);
}

int sol_attn_dense_forward(const void* q, const void* k, const void* v, void* out, int B, int H,
                           int N, int D, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return SOL_ATTN_OK;
  if (st != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  return launch_attend(q, k, v, out, nullptr, B, H, N, D, -INFINITY, 0, nullptr, true,
                       static_cast<cudaStream_t>(stream));
}

int sol_attn_forward_host(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int N, int D, int block, float tau, int prefix_len, int heads_per_chunk,
                          void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if (heads_per_chunk < 0) return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int BH = B * H;  // B*H*N fits in int (check_shape), so B*H does
  // Default chunk: about 8 MiB of each tensor (one head at N = 32768,
  // D = 128), enough for full-speed copies while keeping the pipeline's
  // fill and drain short.
  const size_t seq_bytes = static_cast<size_t>(N) * D * 2;
  const int hc = heads_per_chunk > 0
                     ? std::min(heads_per_chunk, BH)
                     : static_cast<int>(std::min<size_t>(BH, std::max<size_t>(1, ((8u << 20) + seq_bytes - 1) / seq_bytes)));
  const int nchunks = (BH + hc - 1) / hc;
  const int nbuf = std::min(3, nchunks);
  const size_t seq_elems = static_cast<size_t>(N) * D;
  const size_t tensor_bytes = round256(static_cast<size_t>(hc) * seq_elems * 2);
  const size_t set_bytes = 4 * tensor_bytes;  // q, k, v, out of one chunk
  const size_t ws_bytes = sol_attn_workspace_bytes(1, hc, N, D, nullptr);

  uint8_t* dev = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&dev), nbuf * set_bytes + ws_bytes, s) != cudaSuccess)
    return SOL_ATTN_ERR_CUDA;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr, ev_in[3] = {}, ev_out[3] = {}, ev_free[3] = {};
  bool ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming) == cudaSuccess;
  for (int b = 0; ok && b < nbuf; ++b)
    ok = cudaEventCreateWithFlags(&ev_in[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_out[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_free[b], cudaEventDisableTiming) == cudaSuccess;
  // The copy streams start after the allocation and any earlier work on `stream`.
  ok = ok && cudaEventRecord(ev_start, s) == cudaSuccess &&
       cudaStreamWaitEvent(h2d, ev_start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(d2h, ev_start, 0) == cudaSuccess;
  const Workspace w = split_workspace(dev + nbuf * set_bytes, 1, hc, N, D);
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* ho = static_cast<uint8_t*>(out);
  st = SOL_ATTN_OK;
  for (int c = 0; ok && st == SOL_ATTN_OK && c < nchunks; ++c) {
    const int b = c % nbuf;
    const int heads = std::min(hc, BH - c * hc);
    const size_t off = static_cast<size_t>(c) * hc * seq_elems * 2, bytes = heads * seq_elems * 2;
    uint8_t* dq = dev + b * set_bytes;
    uint8_t* dk = dq + tensor_bytes;
    uint8_t* dv = dk + tensor_bytes;
    uint8_t* dout = dv + tensor_bytes;
    // Buffer set b is free once the copy-back of chunk c - nbuf has finished.
    if (c >= nbuf) ok = cudaStreamWaitEvent(h2d, ev_free[b], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dq, hq + off, bytes, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaMemcpyAsync(dk, hk + off, bytes, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaMemcpyAsync(dv, hv + off, bytes, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaEventRecord(ev_in[b], h2d) == cudaSuccess && cudaStreamWaitEvent(s, ev_in[b], 0) == cudaSuccess;
    if (!ok) break;
    st = launch_pool(dq, dk, dv, w, 1, heads, N, D, s);
    if (st == SOL_ATTN_OK)
      st = launch_attend(dq, dk, dv, dout, &w, 1, heads, N, D, tau, prefix_len, nullptr, false, s);
    ok = st == SOL_ATTN_OK && cudaEventRecord(ev_out[b], s) == cudaSuccess &&
         cudaStreamWaitEvent(d2h, ev_out[b], 0) == cudaSuccess &&
         cudaMemcpyAsync(ho + off, dout, bytes, cudaMemcpyDeviceToHost, d2h) == cudaSuccess &&
         cudaEventRecord(ev_free[b], d2h) == cudaSuccess;
  }
  // Whatever happened above, `stream` resumes only after both copy streams
  // have drained (h2d's tail is folded into d2h), and only then is the
  // scratch released.  If that ordering cannot be enqueued, wait here.
  const bool tail = ev_start && ev_done && h2d && d2h && cudaEventRecord(ev_start, h2d) == cudaSuccess &&
                    cudaStreamWaitEvent(d2h, ev_start, 0) == cudaSuccess &&
                    cudaEventRecord(ev_done, d2h) == cudaSuccess &&
                    cudaStreamWaitEvent(s, ev_done, 0) == cudaSuccess;
  if (!tail) {
    if (h2d) cudaStreamSynchronize(h2d);
    if (d2h) cudaStreamSynchronize(d2h);
    ok = false;
  }
  if (cudaFreeAsync(dev, s) != cudaSuccess) ok = false;
  // Streams and events are released by the runtime once their work completes.
  for (int b = 0; b < 3; ++b) {
    if (ev_in[b]) cudaEventDestroy(ev_in[b]);
    if (ev_out[b]) cudaEventDestroy(ev_out[b]);
    if (ev_free[b]) cudaEventDestroy(ev_free[b]);
  }
  if (ev_start) cudaEventDestroy(ev_start);
  if (ev_done) cudaEventDestroy(ev_done);
  if (h2d) cudaStreamDestroy(h2d);
  if (d2h) cudaStreamDestroy(d2h);
  if (st != SOL_ATTN_OK) return st;
  return ok ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

int sol_attn_qknorm_rope_pool(const void* q_in, const void* k_in, const void* v, const float* q_weight,
                              const float* k_weight, void* q_out, void* k_out, void* workspace, int B, int H,
                              int N, int D, int rope_dims, float eps, float rope_base, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return SOL_ATTN_OK;
  if (st != SOL_ATTN_OK) return st;
  if (!q_in || !k_in || !q_out || !k_out || !q_weight || !k_weight || !aligned16(q_in) || !aligned16(k_in) ||
      !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_weight) || !aligned16(k_weight))
    return SOL_ATTN_ERR_INVALID_ARG;
  if (workspace != nullptr &&
      (!v || !aligned16(v) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return SOL_ATTN_ERR_INVALID_ARG;
  const bool pow2 = rope_dims > 0 && ((rope_dims / 16) & (rope_dims / 16 - 1)) == 0;
  if (rope_dims < 0 || rope_dims > D || rope_dims % 16 != 0 || (rope_dims > 0 && !pow2))
    return SOL_ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps <= 0.f || !std::isfinite(rope_base) || rope_base <= 1.f)
    return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  sol::PrepParams pp{};
  pp.q_in = static_cast<const __nv_bfloat16*>(q_in);
  pp.k_in = static_cast<const __nv_bfloat16*>(k_in);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.wq = q_weight;
  pp.wk = k_weight;
  pp.q_out = static_cast<__nv_bfloat16*>(q_out);
  pp.k_out = static_cast<__nv_bfloat16*>(k_out);
  if (workspace != nullptr) {
    const Workspace w = split_workspace(workspace, B, H, N, D);
    pp.pool = sol::PoolOut{w.qbar, w.kbar, w.kbar_bf16, w.vbar_bf16};
  }
  pp.M = N / SOL_ATTN_BLOCK;
  pp.rope_dims = rope_dims;
  pp.eps = eps;
  for (int i = 0; i < rope_dims / 2; ++i)
    pp.inv_freq[i] = std::pow(static_cast<double>(rope_base), -2.0 * i / rope_dims);
  const unsigned nblk = static_cast<unsigned>(static_cast<long long>(B) * H * pp.M);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (workspace != nullptr) {
    dim3 grid(nblk, 3);
    if (D == 128) sol::prep_kernel<128, true><<<grid, 128, 0, s>>>(pp);
    else sol::prep_kernel<64, true><<<grid, 128, 0, s>>>(pp);
  } else {
    dim3 grid(nblk, 2);
    if (D == 128) sol::prep_kernel<128, false><<<grid, 128, 0, s>>>(pp);
    else sol::prep_kernel<64, false><<<grid, 128, 0, s>>>(pp);
  }
  return cudaGetLastError() == cudaSuccess ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

int sol_attn_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SOL_ATTN_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, sol::g_sol_attn_error, sizeof(int)) != cudaSuccess)
    return SOL_ATTN_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(sol::g_sol_attn_error, &zero, sizeof(int)) != cudaSuccess)
      return SOL_ATTN_ERR_CUDA;
    return SOL_ATTN_ERR_DEVICE_TIMEOUT;
  }
  return SOL_ATTN_OK;
}

const char* sol_attn_status_string(int status) {
  switch (status) {
    case SOL_ATTN_OK: return "SOL_ATTN_OK";
    case SOL_ATTN_ERR_INVALID_ARG: return "SOL_ATTN_ERR_INVALID_ARG";
    case SOL_ATTN_ERR_UNSUPPORTED: return "SOL_ATTN_ERR_UNSUPPORTED";
    case SOL_ATTN_ERR_ARCH: return "SOL_ATTN_ERR_ARCH";
    case SOL_ATTN_ERR_CUDA: return "SOL_ATTN_ERR_CUDA";
    case SOL_ATTN_ERR_DEVICE_TIMEOUT: return "SOL_ATTN_ERR_DEVICE_TIMEOUT";
    default: return "SOL_ATTN_ERR_UNKNOWN";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// 8-bit (E4M3) forward: the same operator on E4M3 inputs with per-tensor
// scales, the exact-block and correction products on kind::f8f6f4 tensor
// cores, P rounded to E4M3.
namespace {

int launch_attend_e4m3(const void* q, const void* k, const void* v, void* out, const Workspace& w, int B,
                       int H, int N, float tau, int prefix_len, float q_scale, float k_scale, float v_scale,
                       const sol_attn_opts* o, cudaStream_t s) {
  constexpr int D = 128;
  const int M = N / SOL_ATTN_BLOCK;
  const uint64_t rows = static_cast<uint64_t>(B) * H * N;
  const uint64_t prows = static_cast<uint64_t>(B) * H * M;
  CUtensorMap mq, mk, mv, mkb, mvb;
  if (!make_map_u8(&mq, q, rows, D) || !make_map_u8(&mk, k, rows, D) || !make_map_u8(&mv, v, rows, D) ||
      !make_map_u8(&mkb, w.kbar_bf16, prows, D) || !make_map_u8(&mvb, w.vbar_bf16, prows, D))
    return SOL_ATTN_ERR_CUDA;
  sol::AttnParams p{};
  p.B = B;
  p.H = H;
  p.N = N;
  p.M = M;
  p.P = prefix_len / SOL_ATTN_BLOCK;
  p.tiles_per_head = (M + 1) / 2;
  p.tau = tau;
  const float scale = (o != nullptr && o->softmax_scale > 0.f) ? o->softmax_scale : 1.0f / std::sqrt(128.0f);
  p.scale = scale;                                               // router: real-domain pooled values
  p.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;  // logits of raw E4M3 products
  p.out_scale = v_scale;
  p.qbar = w.qbar;
  p.kbar = w.kbar;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.debug_mask = o ? o->debug_mask : nullptr;
  p.kept_pairs = o ? o->kept_pairs : nullptr;
  p.exact_pairs = o ? o->exact_pairs : nullptr;
  const unsigned tms = (o != nullptr && o->timeout_ms > 0) ? o->timeout_ms : 1000u;
  p.timeout_ns = static_cast<uint64_t>(tms) * 1000000ull;
  p.skip_first_k_arrival = o ? o->test_skip_first_k_load : 0;
  p.budget = o ? o->budget_blocks : 0;
  p.correct = !(o != nullptr && o->skip_correction != 0);
  const long long tiles = static_cast<long long>(B) * H * p.tiles_per_head;
  sol::sol_attn_fwd_kernel<128, false, true><<<dim3(static_cast<unsigned>(tiles)), sol::kThreads,
                                               sol::SmemPlan<128, 1>::kAlloc, s>>>(mq, mk, mv, mkb, mvb, p);
  return cudaGetLastError() == cudaSuccess ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

bool good_scale(float x) { return std::isfinite(x) && x > 0.f; }

int check_scales(float q_scale, float k_scale, float v_scale) {
  return good_scale(q_scale) && good_scale(k_scale) && good_scale(v_scale) ? SOL_ATTN_OK : SOL_ATTN_ERR_INVALID_ARG;
}

int launch_pool_e4m3(const void* q, const void* k, const void* v, const Workspace& w, int B, int H, int N,
                     float q_scale, float k_scale, cudaStream_t s) {
  const unsigned nblk = static_cast<unsigned>(static_cast<long long>(B) * H * (N / SOL_ATTN_BLOCK));
  sol::PoolOutE4M3 po{w.qbar, w.kbar, reinterpret_cast<uint8_t*>(w.kbar_bf16),
                      reinterpret_cast<uint8_t*>(w.vbar_bf16), q_scale, k_scale};
  sol::pool_kernel_e4m3<128><<<dim3(nblk, 3), 128, 0, s>>>(static_cast<const uint8_t*>(q),
                                                          static_cast<const uint8_t*>(k),
                                                          static_cast<const uint8_t*>(v), po);
  return cudaGetLastError() == cudaSuccess ? SOL_ATTN_OK : SOL_ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int sol_attn_pool_fp8(const void* q, const void* k, const void* v, void* workspace, int B, int H, int N, int D,
                      float q_scale, float k_scale, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return SOL_ATTN_OK;
  if (st != SOL_ATTN_OK) return st;
  if (D != 128) return SOL_ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !workspace || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_scales(q_scale, k_scale, 1.0f)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  return launch_pool_e4m3(q, k, v, split_workspace(workspace, B, H, N, D), B, H, N, q_scale, k_scale,
                          static_cast<cudaStream_t>(stream));
}

int sol_attn_attend_fp8(const void* q, const void* k, const void* v, void* out, const void* workspace, int B,
                        int H, int N, int D, int block, float tau, int prefix_len, float q_scale, float k_scale,
                        float v_scale, const sol_attn_opts* opts, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if (D != 128) return SOL_ATTN_ERR_UNSUPPORTED;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SOL_ATTN_ERR_INVALID_ARG;
  if ((st = check_scales(q_scale, k_scale, v_scale)) != SOL_ATTN_OK) return st;
  if ((st = check_opts(opts)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  return launch_attend_e4m3(q, k, v, out, split_workspace(workspace, B, H, N, D), B, H, N, tau, prefix_len,
                            q_scale, k_scale, v_scale, opts, static_cast<cudaStream_t>(stream));
}

int sol_attn_forward_fp8(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int D,
                         int block, float tau, int prefix_len, float q_scale, float k_scale, float v_scale,
                         const sol_attn_opts* opts, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if (D != 128) return SOL_ATTN_ERR_UNSUPPORTED;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if ((st = check_scales(q_scale, k_scale, v_scale)) != SOL_ATTN_OK) return st;
  if ((st = check_opts(opts)) != SOL_ATTN_OK) return st;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = sol_attn_workspace_bytes(B, H, N, D, nullptr);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, s) != cudaSuccess) return SOL_ATTN_ERR_CUDA;
  const Workspace w = split_workspace(ws, B, H, N, D);
  st = launch_pool_e4m3(q, k, v, w, B, H, N, q_scale, k_scale, s);
  if (st == SOL_ATTN_OK)
    st = launch_attend_e4m3(q, k, v, out, w, B, H, N, tau, prefix_len, q_scale, k_scale, v_scale, opts, s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && st == SOL_ATTN_OK) st = SOL_ATTN_ERR_CUDA;
  return st;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward.
//
// Some callers cannot call cudaMalloc while they run attention: a runtime
// that reserves all device memory up front and forbids later allocation, an
// inference server that must not let an allocator lock or fragment memory
// between requests, or code running where the CUDA allocator may not be
// entered.  sol_attn_forward_noalloc serves them.  It uses a fixed scratch
// array compiled into this library instead of cudaMallocAsync, and it calls
// no cudaMalloc, cudaFree or other allocating routine.
//
// The scratch array is a file-scope __device__ array of
// SOL_ATTN_NOALLOC_MAX_WORKSPACE bytes.  Every GPU that loads the library
// holds it until the process exits.  Host code cannot use the array's name
// as a device address (on the host it names a stand-in), so the first call
// on each device, with that device current, looks the address up with
// cudaGetSymbolAddress and caches it.  Make that first call before any
// stream capture.
//
// Every call shares the one array, so two calls whose kernels overlap on the
// GPU (different streams, or different host threads) race on it.  Nothing
// in it must start at zero: the pooling kernel writes every byte the
// attention kernel reads, so the previous call's contents never leak into a
// result.
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[SOL_ATTN_NOALLOC_MAX_WORKSPACE];

struct NoAllocScratch {
  std::once_flag once;
  void* ptr = nullptr;
  int status = SOL_ATTN_ERR_CUDA;
};
NoAllocScratch g_noalloc[kMaxDevices];

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SOL_ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SOL_ATTN_ERR_UNSUPPORTED;
  NoAllocScratch& s = g_noalloc[dev];
  std::call_once(s.once, [&] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess && p != nullptr) {
      s.ptr = p;
      s.status = SOL_ATTN_OK;
    }
  });
  *out = s.ptr;
  return s.status;
}

}  // namespace

extern "C" int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out,
                                        int B, int H, int N, int D, int block, float tau,
                                        int prefix_len, void* stream) {
  int st = check_shape(B, H, N, D);
  if (st == -1) return check_route_args(block, tau, prefix_len, N);
  if (st != SOL_ATTN_OK) return st;
  if ((st = check_route_args(block, tau, prefix_len, N)) != SOL_ATTN_OK) return st;
  if ((st = check_io(q, k, v, out)) != SOL_ATTN_OK) return st;
  if (sol_attn_workspace_bytes(B, H, N, D, nullptr) > SOL_ATTN_NOALLOC_MAX_WORKSPACE)
    return SOL_ATTN_ERR_UNSUPPORTED;
  if ((st = check_device()) != SOL_ATTN_OK) return st;
  void* ws = nullptr;
  if ((st = noalloc_scratch(&ws)) != SOL_ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Workspace w = split_workspace(ws, B, H, N, D);
  st = launch_pool(q, k, v, w, B, H, N, D, s);
  if (st == SOL_ATTN_OK)
    st = launch_attend(q, k, v, out, &w, B, H, N, D, tau, prefix_len, nullptr, false, s);
  return st;
}
