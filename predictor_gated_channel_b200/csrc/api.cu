// api.cu -- the extern "C" entry points of libsfn: argument validation,
// scratch layout and kernel dispatch.  Every check happens before anything
// is enqueued, so an error status means nothing was written.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <utility>
#include <vector>

#include "sfn_internal.cuh"

namespace sfn {

// The library's device error word (bits kDevErr*), set by kernels whose
// bounded waits give up or whose index checks fail.
__device__ unsigned g_sfn_device_error;

namespace {
std::atomic<uint64_t> g_launches{0};
std::mutex g_dev_mu;
DeviceInfo g_dev_cache[64];

// Shape limits of the built kernels (shared-memory staging of x, h).
constexpr int kMaxD = 8192;
constexpr int kMaxR = 2048;
constexpr int kMaxDi = 1 << 24;
constexpr size_t kStageBudget = 96 * 1024;  // bytes of x rows staged per CTA
// The few-token gate/up/down kernel spreads each token over this many CTAs
// (divided among the tokens); fixed so the scratch size does not depend on
// the device.  148 = the SM count of a B200.
constexpr int kPlanSms = 148;

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// ---- optional per-stage timing (sfn_timing_begin / sfn_timing_end)
struct TimingRec {
  int stage;
  cudaEvent_t start, stop;
};
std::mutex g_tmu;
std::atomic<bool> g_timing{false};
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Run one launcher; when timing is on, bracket it with events on `st`.
template <class F>
cudaError_t timed(int stage, cudaStream_t st, F &&launch) {
  if (!g_timing.load(std::memory_order_relaxed)) return launch();
  std::lock_guard<std::mutex> lock(g_tmu);
  cudaEvent_t a = take_event(), b = take_event();
  if (a) cudaEventRecord(a, st);
  cudaError_t e = launch();
  if (b) cudaEventRecord(b, st);
  if (a && b) g_recs.push_back({stage, a, b});
  return e;
}

int pow2_tokens(int64_t T, int cap) {
  int tt = 1;
  while (tt < cap && tt < T) tt *= 2;
  return tt;
}
}  // namespace

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

cudaError_t ensure_smem_limit(const void *kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  struct Key {
    const void *k;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Key> done;
  std::lock_guard<std::mutex> lock(mu);
  for (const Key &kk : done)
    if (kk.k == kernel && kk.dev == dev && kk.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.push_back({kernel, dev, bytes});
  return e;
}

bool device_info(DeviceInfo *out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo &c = g_dev_cache[dev];
  if (c.device != dev) {
    int major = 0, sms = 0, smem = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
      return false;
    if (major != 10) return false;  // the library is built for sm_100a only
    void *err = nullptr;
    if (cudaGetSymbolAddress(&err, g_sfn_device_error) != cudaSuccess) return false;
    c.err = static_cast<unsigned *>(err);
    c.num_sms = sms;
    c.max_smem_optin = smem;
    c.device = dev;
  }
  *out = c;
  return true;
}

int pred_tokens_per_cta(const FwdShape &s) {
  int tt = pow2_tokens(s.T, 8);
  while (tt > 1 && (size_t)tt * s.d * sizeof(float) > kStageBudget) tt /= 2;
  return tt;
}

GatherPlan plan_gather(const FwdShape &s) {
  GatherPlan p{};
  p.tt_h = pred_tokens_per_cta(s);
  p.tt_p = pow2_tokens(s.T, 8);
  p.cpt = ffn_ctas_per_token(s, kPlanSms);
  size_t off = 0;
  p.off_h = off;
  off = align_up(off + (size_t)s.T * s.r * sizeof(float), 256);
  p.off_idx = off;
  off = align_up(off + (size_t)s.T * s.d_s * sizeof(int), 256);
  p.off_sig = off;
  off = align_up(off + (size_t)s.T * s.d_s * sizeof(float), 256);
  p.off_part = off;
  off = align_up(off + (size_t)s.T * p.cpt * s.d * sizeof(float), 256);
  p.total = off;
  return p;
}

}  // namespace sfn

using namespace sfn;

namespace {
thread_local const char *t_last_error = "no error";

sfn_status check_shape(int64_t T, int d, int d_i, int r, int bank, int k) {
  if (T < 0 || d <= 0 || d_i <= 0 || r <= 0) return SFN_ERR_INVALID_VALUE;
  if (bank < 1 || bank > 64 || k < 1 || k > bank || d_i % bank != 0)
    return SFN_ERR_INVALID_VALUE;
  return SFN_OK;
}

sfn_status check_limits(int d, int d_i, int r) {
  if (d > kMaxD || r > kMaxR || d_i > kMaxDi) return SFN_ERR_UNSUPPORTED;
  return SFN_OK;
}

sfn_status check_rows(int d, int r, bool bf16) {
  const int elt = bf16 ? 2 : 4;
  if ((d * elt) % 16 != 0 || (r * elt) % 16 != 0) return SFN_ERR_MISALIGNED;
  return SFN_OK;
}

FwdShape make_shape(int64_t T, int d, int d_i, int r, int bank, int k, bool bf16) {
  FwdShape s;
  s.T = T;
  s.d = d;
  s.d_i = d_i;
  s.r = r;
  s.bank = bank;
  s.k = k;
  s.n_banks = d_i / bank;
  s.d_s = s.n_banks * k;
  s.bf16 = bf16;
  return s;
}

sfn_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SFN_OK;
  t_last_error = cudaGetErrorString(e);
  cudaGetLastError();  // clear a sticky launch error of our own making
  return SFN_ERR_CUDA;
}

sfn_status predict_impl(const void *x, const void *A, const void *B, float *logits, int64_t T,
                        int d, int d_i, int r, bool bf16, cudaStream_t st) {
  sfn_status s0 = check_shape(T, d, d_i, r, 1, 1);
  if (s0 != SFN_OK) return s0;
  if ((s0 = check_limits(d, d_i, r)) != SFN_OK) return s0;
  if ((s0 = check_rows(d, r, bf16)) != SFN_OK) return s0;
  if (T == 0) return SFN_OK;
  if (!x || !A || !B || !logits) return SFN_ERR_INVALID_VALUE;
  if (!aligned(x, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(logits, 16))
    return SFN_ERR_MISALIGNED;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  FwdShape s = make_shape(T, d, d_i, r, 64, 16, bf16);
  const bool tc = tc_shape_ok(s) && T >= 1024;
  const size_t need = tc ? (size_t)T * 2 * r * 2 : (size_t)T * r * sizeof(float);
  void *scratch = nullptr;
  if (cudaMallocAsync(&scratch, need, st) != cudaSuccess)
    return cuda_status(cudaErrorMemoryAllocation);
  cudaError_t e;
  if (tc) {
    uint16_t *h2 = static_cast<uint16_t *>(scratch);
    e = timed(SFN_STAGE_TC_H, st,
              [&] { return launch_tc_h(s, dev, x, A, h2, nullptr, 1, st); });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_TC_LOGITS_TOPK, st,
                [&] { return launch_tc_logits(s, dev, h2, B, logits, nullptr, nullptr, st); });
  } else {
    GatherPlan p = plan_gather(s);
    float *h = static_cast<float *>(scratch);
    const size_t b_bytes = (size_t)s.d_i * s.r * (s.bf16 ? 2 : 4);
    e = timed(SFN_STAGE_PRED_H, st,
              [&] { return launch_pred_h(s, p.tt_h, x, A, h, false, st, B, b_bytes); });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_LOGITS_TOPK, st, [&] {
        return launch_logits_topk(s, p.tt_p, h, B, logits, nullptr, nullptr, nullptr, dev.err,
                                  st);
      });
  }
  cudaError_t ef = cudaFreeAsync(scratch, st);
  if (e == cudaSuccess) e = ef;
  return cuda_status(e);
}

// Fewest tokens for which the automatic choice takes the tensor-core path.
// The CUDA-core path streams each token's kept rows separately (T x 88 MB for
// the 4096 x 14336 layer), bound by what each SM can pull; the tensor path
// reads the union of the tokens' kept rows once, with dense tiles.  Measured
// graph-replayed step times on that layer (bf16, B200), CUDA-core vs tensor:
// T = 4: 67 vs 86 us; T = 5: 86 vs 87 us; T = 6: 96 vs 87 us; T = 8: 114 vs
// 87 us.
constexpr int64_t kTcMinTokens = 6;
bool use_tensor_path(const FwdShape &s, sfn_path path) {
  if (path == SFN_PATH_CUDA_CORE) return false;
  if (!tc_shape_ok(s)) return false;
  return path == SFN_PATH_TENSOR || s.T >= kTcMinTokens;
}

size_t workspace_for(const FwdShape &s) {
  size_t need = plan_gather(s).total;
  if (tc_shape_ok(s)) need = std::max(need, plan_tc(s).total);
  return need;
}

sfn_status forward_impl(const void *x, const void *A, const void *B, const void *Wg,
                        const void *Wu, const void *Wd, void *y, uint64_t *mask, int64_t T,
                        int d, int d_i, int r, int bank, int k, bool bf16, sfn_path path,
                        void *ws, size_t ws_bytes, bool own_ws, cudaStream_t st,
                        bool y_f32 = false) {
  sfn_status s0 = check_shape(T, d, d_i, r, bank, k);
  if (s0 != SFN_OK) return s0;
  if (path != SFN_PATH_AUTO && path != SFN_PATH_CUDA_CORE && path != SFN_PATH_TENSOR)
    return SFN_ERR_INVALID_VALUE;
  if ((s0 = check_limits(d, d_i, r)) != SFN_OK) return s0;
  if ((s0 = check_rows(d, r, bf16)) != SFN_OK) return s0;
  if (T == 0) return SFN_OK;
  if (!x || !A || !B || !Wg || !Wu || !Wd || !y) return SFN_ERR_INVALID_VALUE;
  if (!aligned(x, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(Wg, 16) ||
      !aligned(Wu, 16) || !aligned(Wd, 16) || !aligned(y, 16) ||
      (mask && !aligned(mask, 8)))
    return SFN_ERR_MISALIGNED;
  FwdShape s = make_shape(T, d, d_i, r, bank, k, bf16);
  if (path == SFN_PATH_TENSOR && !tc_shape_ok(s)) return SFN_ERR_UNSUPPORTED;
  const bool tc = use_tensor_path(s, path);
  if (!tc && !ffn_shape_ok(s)) return SFN_ERR_UNSUPPORTED;
  const size_t need = tc ? plan_tc(s).total : plan_gather(s).total;
  if (!own_ws && (ws == nullptr || !aligned(ws, 256) || ws_bytes < need))
    return SFN_ERR_WORKSPACE;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  if (own_ws && cudaMallocAsync(&ws, need, st) != cudaSuccess)
    return cuda_status(cudaErrorMemoryAllocation);
  char *w = static_cast<char *>(ws);
  cudaError_t e = cudaSuccess;
  if (tc) {
    const TcPlan p = plan_tc(s);
    uint16_t *h2 = reinterpret_cast<uint16_t *>(w + p.off_h2);
    float *sig = reinterpret_cast<float *>(w + p.off_sig);
    uint16_t *act = reinterpret_cast<uint16_t *>(w + p.off_act);
    uint64_t *m = mask ? mask : reinterpret_cast<uint64_t *>(w + p.off_mask);
    if (p.hsplit > 1) {
      // few 128-token tiles: split K, then sum the fp32 partials and split
      // the sum into the bf16 hi/lo operand of the logits GEMM
      float *hpart = reinterpret_cast<float *>(w + p.off_hpart);
      e = timed(SFN_STAGE_TC_H, st,
                [&] { return launch_tc_h(s, dev, x, A, h2, hpart, p.hsplit, st); });
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_REDUCE, st, [&] {
          return launch_reduce_partials(s, p.hsplit, hpart, h2, st, ReduceOut::kSplitH);
        });
    } else {
      e = timed(SFN_STAGE_TC_H, st,
                [&] { return launch_tc_h(s, dev, x, A, h2, nullptr, 1, st); });
    }
    if (tc_fused_gateup_ok(s)) {
      // one token tile: logits, bank top-k and the masked gate/up in one kernel
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_TC_GATEUP, st, [&] {
          return launch_tc_logits_gateup(s, dev, h2, B, x, Wg, Wu, mask, act, st);
        });
    } else {
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_TC_LOGITS_TOPK, st,
                  [&] { return launch_tc_logits(s, dev, h2, B, nullptr, m, sig, st); });
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_TC_GATEUP, st,
                  [&] { return launch_tc_gateup(s, dev, x, Wg, Wu, m, sig, act, st); });
    }
    if (p.ksplit > 1) {
      float *part = reinterpret_cast<float *>(w + p.off_part);
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_TC_DOWN, st,
                  [&] { return launch_tc_down(s, dev, act, Wd, part, p.ksplit, st); });
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_REDUCE, st, [&] {
          return launch_reduce_partials(s, p.ksplit, part, y, st,
                                        y_f32 ? ReduceOut::kYF32 : ReduceOut::kY);
        });
    } else if (e == cudaSuccess) {
      e = timed(SFN_STAGE_TC_DOWN, st,
                [&] { return launch_tc_down(s, dev, act, Wd, y, 1, st, y_f32); });
    }
  } else {
    const GatherPlan p = plan_gather(s);
    float *h = reinterpret_cast<float *>(w + p.off_h);
    int *sel_idx = reinterpret_cast<int *>(w + p.off_idx);
    float *sel_sig = reinterpret_cast<float *>(w + p.off_sig);
    float *partial = reinterpret_cast<float *>(w + p.off_part);
    const size_t b_bytes = (size_t)s.d_i * s.r * (s.bf16 ? 2 : 4);
    e = timed(SFN_STAGE_PRED_H, st,
              [&] { return launch_pred_h(s, p.tt_h, x, A, h, false, st, B, b_bytes); });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_LOGITS_TOPK, st, [&] {
        return launch_logits_topk(s, p.tt_p, h, B, nullptr, mask, sel_idx, sel_sig, dev.err, st);
      });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_FFN, st, [&] {
        return launch_ffn(s, p.cpt, x, sel_idx, sel_sig, Wg, Wu, Wd, partial, dev.err, st);
      });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_REDUCE, st,
                [&] {
                  return launch_reduce_partials(s, p.cpt, partial, y, st,
                                                y_f32 ? ReduceOut::kYF32 : ReduceOut::kY);
                });
  }
  if (own_ws) {
    cudaError_t ef = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = ef;
  }
  return cuda_status(e);
}

// Scratch of the Dense-4x comparison: act [T][d_i] bf16, a mask, and the
// down GEMM's split-K partials.
struct Dense4xPlan {
  int ksplit;
  size_t off_act, off_mask, off_part, total;
};
Dense4xPlan plan_dense4x(const FwdShape &s) {
  Dense4xPlan p{};
  p.ksplit = tc_down_splits(s, kPlanSms);
  size_t off = 0;
  p.off_act = off;
  off = align_up(off + (size_t)s.T * s.d_i * 2, 256);
  p.off_mask = off;
  off = align_up(off + (size_t)s.T * s.n_banks * 8, 256);
  p.off_part = off;
  if (p.ksplit > 1) off = align_up(off + (size_t)s.T * p.ksplit * s.d * 4, 256);
  p.total = off;
  return p;
}

}  // namespace

extern "C" {

const char *sfn_status_string(sfn_status s) {
  switch (s) {
    case SFN_OK: return "SFN_OK: success";
    case SFN_ERR_INVALID_VALUE: return "SFN_ERR_INVALID_VALUE: invalid shape, k, bank or pointer";
    case SFN_ERR_MISALIGNED: return "SFN_ERR_MISALIGNED: pointer or row not 16-byte aligned";
    case SFN_ERR_UNSUPPORTED: return "SFN_ERR_UNSUPPORTED: shape outside the built kernels' limits";
    case SFN_ERR_WORKSPACE: return "SFN_ERR_WORKSPACE: scratch missing, misaligned or too small";
    case SFN_ERR_CUDA: return "SFN_ERR_CUDA: CUDA call or launch failed";
  }
  return "unknown sfn_status";
}

int sfn_abi_version(void) { return 2; }

const char *sfn_last_error_string(void) { return t_last_error; }

uint64_t sfn_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

sfn_status sfn_predict(const void *x, const void *A, const void *B, float *logits, int64_t T,
                       int d, int d_i, int r, sfn_stream_t stream) {
  return predict_impl(x, A, B, logits, T, d, d_i, r, true, (cudaStream_t)stream);
}

sfn_status sfn_predict_f32(const float *x, const float *A, const float *B, float *logits,
                           int64_t T, int d, int d_i, int r, sfn_stream_t stream) {
  return predict_impl(x, A, B, logits, T, d, d_i, r, false, (cudaStream_t)stream);
}

sfn_status sfn_bank_topk(const float *logits, uint64_t *mask, int64_t T, int d_i, int bank,
                         int k, sfn_stream_t stream) {
  if (T < 0 || d_i <= 0 || bank < 1 || bank > 64 || k < 1 || k > bank || d_i % bank != 0)
    return SFN_ERR_INVALID_VALUE;
  if (d_i > kMaxDi) return SFN_ERR_UNSUPPORTED;
  if (T == 0) return SFN_OK;
  if (!logits || !mask) return SFN_ERR_INVALID_VALUE;
  if (!aligned(logits, 4) || !aligned(mask, 8)) return SFN_ERR_MISALIGNED;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  return cuda_status(timed(SFN_STAGE_BANK_TOPK, st, [&] {
    return launch_bank_topk(logits, mask, T, d_i, bank, k, st);
  }));
}

size_t sfn_workspace_bytes(int64_t T, int d, int d_i, int r, int bank, int k,
                           sfn_dtype dtype) {
  if (dtype != SFN_DTYPE_BF16 && dtype != SFN_DTYPE_F32) return 0;
  if (check_shape(T, d, d_i, r, bank, k) != SFN_OK || T == 0) return 0;
  if (check_limits(d, d_i, r) != SFN_OK) return 0;
  return workspace_for(make_shape(T, d, d_i, r, bank, k, dtype == SFN_DTYPE_BF16));
}

sfn_status sfn_sparse_ffn_forward(const void *x, const void *A, const void *B, const void *Wg,
                                  const void *Wu, const void *Wd, void *y, uint64_t *mask,
                                  int64_t T, int d, int d_i, int r, int bank, int k,
                                  sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, true, SFN_PATH_AUTO,
                      nullptr, 0, true, (cudaStream_t)stream);
}

sfn_status sfn_sparse_ffn_forward_ws(const void *x, const void *A, const void *B,
                                     const void *Wg, const void *Wu, const void *Wd, void *y,
                                     uint64_t *mask, int64_t T, int d, int d_i, int r,
                                     int bank, int k, void *workspace, size_t workspace_bytes,
                                     sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, true, SFN_PATH_AUTO,
                      workspace, workspace_bytes, false, (cudaStream_t)stream);
}

sfn_status sfn_sparse_ffn_forward_path(const void *x, const void *A, const void *B,
                                       const void *Wg, const void *Wu, const void *Wd, void *y,
                                       uint64_t *mask, int64_t T, int d, int d_i, int r,
                                       int bank, int k, sfn_path path, void *workspace,
                                       size_t workspace_bytes, sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, true, path,
                      workspace, workspace_bytes, false, (cudaStream_t)stream);
}

sfn_status sfn_sparse_ffn_forward_partial(const void *x, const void *A, const void *B,
                                          const void *Wg, const void *Wu, const void *Wd,
                                          float *y_partial, uint64_t *mask, int64_t T, int d,
                                          int d_i, int r, int bank, int k, sfn_path path,
                                          void *workspace, size_t workspace_bytes,
                                          sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y_partial, mask, T, d, d_i, r, bank, k, true, path,
                      workspace, workspace_bytes, false, (cudaStream_t)stream, true);
}

sfn_status sfn_sparse_ffn_forward_f32(const float *x, const float *A, const float *B,
                                      const float *Wg, const float *Wu, const float *Wd,
                                      float *y, uint64_t *mask, int64_t T, int d, int d_i,
                                      int r, int bank, int k, sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, false,
                      SFN_PATH_AUTO, nullptr, 0, true, (cudaStream_t)stream);
}

sfn_status sfn_sparse_ffn_forward_f32_ws(const float *x, const float *A, const float *B,
                                         const float *Wg, const float *Wu, const float *Wd,
                                         float *y, uint64_t *mask, int64_t T, int d, int d_i,
                                         int r, int bank, int k, void *workspace,
                                         size_t workspace_bytes, sfn_stream_t stream) {
  return forward_impl(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, false,
                      SFN_PATH_AUTO, workspace, workspace_bytes, false, (cudaStream_t)stream);
}

sfn_status sfn_timing_begin(void) {
  std::lock_guard<std::mutex> lock(g_tmu);
  for (auto &r : g_recs) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_recs.clear();
  g_timing.store(true);
  return SFN_OK;
}

sfn_status sfn_timing_end(double *ms, uint64_t *launches, int n) {
  std::lock_guard<std::mutex> lock(g_tmu);
  g_timing.store(false);
  if (ms)
    for (int i = 0; i < n; ++i) ms[i] = 0.0;
  if (launches)
    for (int i = 0; i < n; ++i) launches[i] = 0;
  sfn_status st = SFN_OK;
  for (auto &r : g_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      st = SFN_ERR_CUDA;
      continue;
    }
    if (r.stage >= 0 && r.stage < n) {
      if (ms) ms[r.stage] += t;
      if (launches) launches[r.stage] += 1;
    }
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_recs.clear();
  if (st != SFN_OK) cudaGetLastError();
  return st;
}

sfn_status sfn_device_errors(unsigned *bits, int clear) {
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaErrorUnknown);
  unsigned v = 0;
  if (cudaMemcpy(&v, dev.err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_status(cudaErrorUnknown);
  if (clear && v != 0 && cudaMemset(dev.err, 0, sizeof v) != cudaSuccess)
    return cuda_status(cudaErrorUnknown);
  if (bits) *bits = v;
  return SFN_OK;
}

size_t sfn_dense4x_workspace_bytes(int64_t T, int d, int d_i, int bank, int k) {
  if (check_shape(T, d, d_i, 64, bank, k) != SFN_OK || T == 0) return 0;
  if (check_limits(d, d_i, 64) != SFN_OK) return 0;
  return plan_dense4x(make_shape(T, d, d_i, 64, bank, k, true)).total;
}

sfn_status sfn_dense4x_forward(const void *x, const void *Wg, const void *Wu, const void *Wd,
                               void *y, uint64_t *mask, int64_t T, int d, int d_i, int bank,
                               int k, void *ws, size_t ws_bytes, sfn_stream_t stream) {
  sfn_status s0 = check_shape(T, d, d_i, 64, bank, k);
  if (s0 != SFN_OK) return s0;
  if ((s0 = check_limits(d, d_i, 64)) != SFN_OK) return s0;
  if ((s0 = check_rows(d, 64, true)) != SFN_OK) return s0;
  FwdShape s = make_shape(T, d, d_i, 64, bank, k, true);
  if (!(bank == 64 && d % 256 == 0 && d_i % 256 == 0)) return SFN_ERR_UNSUPPORTED;
  if (T == 0) return SFN_OK;
  if (!x || !Wg || !Wu || !Wd || !y) return SFN_ERR_INVALID_VALUE;
  if (!aligned(x, 16) || !aligned(Wg, 16) || !aligned(Wu, 16) || !aligned(Wd, 16) ||
      !aligned(y, 16) || (mask && !aligned(mask, 8)))
    return SFN_ERR_MISALIGNED;
  const Dense4xPlan p = plan_dense4x(s);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < p.total) return SFN_ERR_WORKSPACE;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  char *w = static_cast<char *>(ws);
  uint16_t *act = reinterpret_cast<uint16_t *>(w + p.off_act);
  uint64_t *m = mask ? mask : reinterpret_cast<uint64_t *>(w + p.off_mask);
  cudaError_t e = timed(SFN_STAGE_DENSE4X_GATEUP, st, [&] {
    return launch_tc_dense4x_gateup(s, dev, x, Wg, Wu, m, act, st);
  });
  if (p.ksplit > 1) {
    float *part = reinterpret_cast<float *>(w + p.off_part);
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_TC_DOWN, st,
                [&] { return launch_tc_down(s, dev, act, Wd, part, p.ksplit, st); });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_REDUCE, st,
                [&] { return launch_reduce_partials(s, p.ksplit, part, y, st); });
  } else if (e == cudaSuccess) {
    e = timed(SFN_STAGE_TC_DOWN, st, [&] { return launch_tc_down(s, dev, act, Wd, y, 1, st); });
  }
  return cuda_status(e);
}

namespace {
// Scratch of the backward.  tc: logits by the tensor-core kernels (the
// forward's automatic choice for this T), h as bf16 hi | lo halves [T][2r];
// otherwise h float32 plus a bf16 copy.
struct BwdPlan {
  bool tc;
  int hsplit;
  size_t off_h2, off_hpart, off_hf, off_hb, off_P, off_mask, off_tau, off_G, off_U, off_DA,
      off_a, off_dg, off_du, off_dp, off_dH, off_dHb, total;
};

BwdPlan plan_bwd(const FwdShape &s) {
  BwdPlan p{};
  p.tc = use_tensor_path(s, SFN_PATH_AUTO);
  p.hsplit = p.tc ? plan_tc(s).hsplit : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t T = (size_t)s.T, r = (size_t)s.r, di = (size_t)s.d_i, nb = (size_t)s.n_banks;
  p.off_h2 = take(p.tc ? T * 2 * r * 2 : 0);
  p.off_hpart = take(p.tc && p.hsplit > 1 ? T * (size_t)p.hsplit * r * 4 : 0);
  p.off_hf = take(p.tc ? 0 : T * r * 4);
  p.off_hb = take(p.tc ? 0 : T * r * 2);
  p.off_P = take(T * di * 4);
  p.off_mask = take(T * nb * 8);
  p.off_tau = take(T * nb * 4);
  p.off_G = take(T * di * 4);
  p.off_U = take(T * di * 4);
  p.off_DA = take(T * di * 4);
  p.off_a = take(T * di * 2);
  p.off_dg = take(T * di * 2);
  p.off_du = take(T * di * 2);
  p.off_dp = take(T * di * 2);
  p.off_dH = take(T * r * 4);
  p.off_dHb = take(T * r * 2);
  p.total = off;
  return p;
}

sfn_status check_backward(int64_t T, int d, int d_i, int r, int bank, int k, float temp) {
  sfn_status s0 = check_shape(T, d, d_i, r, bank, k);
  if (s0 != SFN_OK) return s0;
  if (!(temp > 0.f) || !std::isfinite(temp)) return SFN_ERR_INVALID_VALUE;
  if ((s0 = check_limits(d, d_i, r)) != SFN_OK) return s0;
  if ((s0 = check_rows(d, r, true)) != SFN_OK) return s0;
  // the tensor-core contractions take N in multiples of 64 (N is d, d_i or r)
  if (d % 64 != 0 || d_i % 64 != 0 || r % 64 != 0 || T > 0x7fffffffLL)
    return SFN_ERR_UNSUPPORTED;
  return SFN_OK;
}
}  // namespace

size_t sfn_backward_workspace_bytes(int64_t T, int d, int d_i, int r, int bank, int k) {
  if (T == 0 || check_backward(T, d, d_i, r, bank, k, 1.f) != SFN_OK) return 0;
  return plan_bwd(make_shape(T, d, d_i, r, bank, k, true)).total;
}

sfn_status sfn_sparse_ffn_backward(const void *x, const void *A, const void *B, const void *Wg,
                                   const void *Wu, const void *Wd, const void *dy,
                                   float temperature, float *dx, float *dA, float *dB,
                                   float *dWg, float *dWu, float *dWd, uint64_t *mask,
                                   int64_t T, int d, int d_i, int r, int bank, int k,
                                   void *ws, size_t ws_bytes, sfn_stream_t stream) {
  sfn_status s0 = check_backward(T, d, d_i, r, bank, k, temperature);
  if (s0 != SFN_OK) return s0;
  if (T == 0) return SFN_OK;
  if (!x || !A || !B || !Wg || !Wu || !Wd || !dy) return SFN_ERR_INVALID_VALUE;
  for (const void *q : {x, A, B, Wg, Wu, Wd, dy, (const void *)dx, (const void *)dA,
                        (const void *)dB, (const void *)dWg, (const void *)dWu,
                        (const void *)dWd})
    if (q && !aligned(q, 16)) return SFN_ERR_MISALIGNED;
  if (mask && !aligned(mask, 8)) return SFN_ERR_MISALIGNED;
  FwdShape s = make_shape(T, d, d_i, r, bank, k, true);
  const BwdPlan p = plan_bwd(s);
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < p.total) return SFN_ERR_WORKSPACE;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  char *w = static_cast<char *>(ws);
  auto F = [&](size_t off) { return reinterpret_cast<float *>(w + off); };
  auto H = [&](size_t off) { return reinterpret_cast<uint16_t *>(w + off); };
  float *P = F(p.off_P), *tau = F(p.off_tau), *G = F(p.off_G), *U = F(p.off_U);
  float *DA = F(p.off_DA), *dH = F(p.off_dH);
  uint16_t *a = H(p.off_a), *dg = H(p.off_dg), *du = H(p.off_du), *dp = H(p.off_dp);
  uint16_t *dHb = H(p.off_dHb);
  uint64_t *m = mask ? mask : reinterpret_cast<uint64_t *>(w + p.off_mask);
  const int Ti = (int)T;

  // 1. the forward's predictor (same kernels as the forward: same logits, same mask)
  const uint16_t *hb;
  int ldh;
  cudaError_t e;
  if (p.tc) {
    uint16_t *h2 = H(p.off_h2);
    if (p.hsplit > 1) {
      float *hpart = F(p.off_hpart);
      e = timed(SFN_STAGE_TC_H, st,
                [&] { return launch_tc_h(s, dev, x, A, h2, hpart, p.hsplit, st); });
      if (e == cudaSuccess)
        e = timed(SFN_STAGE_REDUCE, st, [&] {
          return launch_reduce_partials(s, p.hsplit, hpart, h2, st, ReduceOut::kSplitH);
        });
    } else {
      e = timed(SFN_STAGE_TC_H, st, [&] { return launch_tc_h(s, dev, x, A, h2, nullptr, 1, st); });
    }
    // logits, mask and thresholds from one GEMM epilogue
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_TC_LOGITS_TOPK, st,
                [&] { return launch_tc_logits_tau(s, dev, h2, B, P, m, tau, st); });
    hb = h2;  // the hi halves: bf16(h)
    ldh = 2 * r;
  } else {
    float *hf = F(p.off_hf);
    uint16_t *hbw = H(p.off_hb);
    e = timed(SFN_STAGE_PRED_H, st, [&] {
      return launch_pred_h(s, pred_tokens_per_cta(s), x, A, hf, false, st);
    });
    if (e == cudaSuccess)
      e = timed(SFN_STAGE_LOGITS_TOPK, st, [&] {
        return launch_logits_topk(s, pow2_tokens(T, 8), hf, B, P, nullptr, nullptr, nullptr,
                                  dev.err, st);
      });
    if (e == cudaSuccess) e = launch_f32_to_bf16(hf, hbw, T * r, st);
    hb = hbw;
    ldh = r;
  }
  // 2. mask and thresholds (the tensor-core logits epilogue already wrote them)
  if (e == cudaSuccess && !p.tc)
    e = timed(SFN_STAGE_BWD_TAU, st,
              [&] { return launch_bank_tau(P, m, tau, T, d_i, bank, k, st); });
  // The contractions run on this library's tcgen05 GEMM (bf16 operands,
  // float32 accumulate and output).  gemm(M, N, K, A, lda, a_mn, B, ldb, b_mn,
  // C, ldc, acc): C[M][N] (+)= A B with A [M][K] or [K][M] (a_mn), B [N][K]
  // or [K][N] (b_mn).
  auto gemm = [&](int mm, int nn, int kk, const void *Am, int lda, bool a_mn, const void *Bm,
                  int ldb, bool b_mn, float *C, int ldc, bool acc) {
    return launch_tc_gemm_f32(dev, mm, nn, kk, Am, lda, a_mn, Bm, ldb, b_mn, C, ldc, acc, st);
  };
  // 3. g = Wg x, u = Wu x (every channel) and da = Wd dy, float32 [T][d_i]
  if (e == cudaSuccess)
    e = timed(SFN_STAGE_BWD_GEMM, st, [&] {
      cudaError_t r1 = gemm(Ti, d_i, d, x, d, false, Wg, d, false, G, d_i, false);
      if (r1 == cudaSuccess) r1 = gemm(Ti, d_i, d, x, d, false, Wu, d, false, U, d_i, false);
      if (r1 == cudaSuccess) r1 = gemm(Ti, d_i, d, dy, d, false, Wd, d, false, DA, d_i, false);
      return r1;
    });
  // 4. the chain rule with the surrogate
  if (e == cudaSuccess)
    e = timed(SFN_STAGE_BWD_ELEM, st, [&] {
      return launch_bwd_elem(P, m, tau, G, U, DA, a, dg, du, dp, T, d_i, bank, temperature,
                             st);
    });
  // 5. contractions back to the inputs; the weight gradients contract over
  // the tokens (K = T), with both operands stored token-major
  const bool need_dh = dA != nullptr || dx != nullptr;
  if (e == cudaSuccess)
    e = timed(SFN_STAGE_BWD_GEMM, st, [&] {
      cudaError_t r1 = cudaSuccess;
      // dWd[j][n] = sum_t a[t][j] dy[t][n]
      if (dWd) r1 = gemm(d_i, d, Ti, a, d_i, true, dy, d, true, dWd, d, false);
      // dWg[j][n] = sum_t dg[t][j] x[t][n]; dWu likewise with du
      if (r1 == cudaSuccess && dWg) r1 = gemm(d_i, d, Ti, dg, d_i, true, x, d, true, dWg, d, false);
      if (r1 == cudaSuccess && dWu) r1 = gemm(d_i, d, Ti, du, d_i, true, x, d, true, dWu, d, false);
      // dB[j][m] = sum_t dp[t][j] h[t][m]
      if (r1 == cudaSuccess && dB) r1 = gemm(d_i, r, Ti, dp, d_i, true, hb, ldh, true, dB, r, false);
      // dh[t][m] = sum_j dp[t][j] B[j][m]
      if (r1 == cudaSuccess && need_dh)
        r1 = gemm(Ti, r, d_i, dp, d_i, false, B, r, true, dH, r, false);
      return r1;
    });
  if (e == cudaSuccess && need_dh) e = launch_f32_to_bf16(dH, dHb, T * r, st);
  if (e == cudaSuccess && need_dh)
    e = timed(SFN_STAGE_BWD_GEMM, st, [&] {
      cudaError_t r1 = cudaSuccess;
      // dA[m][n] = sum_t dh[t][m] x[t][n]
      if (dA) r1 = gemm(r, d, Ti, dHb, r, true, x, d, true, dA, d, false);
      // dx = dg Wg + du Wu + dh A, accumulated in float32
      if (r1 == cudaSuccess && dx) {
        r1 = gemm(Ti, d, d_i, dg, d_i, false, Wg, d, true, dx, d, false);
        if (r1 == cudaSuccess) r1 = gemm(Ti, d, d_i, du, d_i, false, Wu, d, true, dx, d, true);
        if (r1 == cudaSuccess) r1 = gemm(Ti, d, r, dHb, r, false, A, d, true, dx, d, true);
      }
      return r1;
    });
  return cuda_status(e);
}

const char *sfn_stage_name(int stage) {
  switch (stage) {
    case SFN_STAGE_PRED_H: return "pred_h";
    case SFN_STAGE_LOGITS_TOPK: return "logits_topk";
    case SFN_STAGE_FFN: return "ffn";
    case SFN_STAGE_REDUCE: return "reduce";
    case SFN_STAGE_TC_H: return "tc_h";
    case SFN_STAGE_TC_LOGITS_TOPK: return "tc_logits_topk";
    case SFN_STAGE_TC_GATEUP: return "tc_gateup";
    case SFN_STAGE_TC_DOWN: return "tc_down";
    case SFN_STAGE_DENSE4X_GATEUP: return "dense4x_gateup";
    case SFN_STAGE_BWD_TAU: return "bwd_tau";
    case SFN_STAGE_BWD_ELEM: return "bwd_elem";
    case SFN_STAGE_BWD_GEMM: return "bwd_gemm";
    case SFN_STAGE_BANK_TOPK: return "bank_topk";
  }
  return "unused";
}

}  // extern "C"
