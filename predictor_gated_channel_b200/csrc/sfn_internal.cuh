// sfn_internal.cuh -- device helpers and host launcher declarations shared by
// the libsfn translation units.  Nothing here is part of the public ABI.
#pragma once
#include <mutex>

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "sfn.h"

namespace sfn {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- elements
// A 16-byte chunk holds kVec elements; both types unpack to float.
struct EltBF16 {
  static constexpr int kVec = 8;
  static constexpr int kBytes = 2;
  __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
  }
};
struct EltF32 {
  static constexpr int kVec = 4;
  static constexpr int kBytes = 4;
  __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

// float -> bf16 bits, round to nearest even (finite inputs; NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Read-only 16-byte load of streamed weights: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_nc16(const void *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Logistic function with CUDA's expf (full-precision library call).
__device__ __forceinline__ float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

// Order-preserving key of a float logit for the bank ranking: a larger logit
// gets a larger key, +0 and -0 share one key, every NaN maps to 0, below the
// key of -inf.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN
  if ((b << 1) == 0u) b = 0u;                      // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Float value of an order key (the inverse of order_key for numbers; -0
// comes back as +0).
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Hard top-k of one bank (bank <= 64) held by a warp: lane l holds the keys
// of channels l (key0) and l + 32 (key1).  Channel i ranks below channel j
// when key_j > key_i, or key_j == key_i and j < i; a channel is kept when
// fewer than k channels rank above it.  Returns the 64-bit keep mask (bit i =
// channel i), identical in every lane.
__device__ __forceinline__ uint64_t warp_bank_topk(uint32_t key0, uint32_t key1, int bank,
                                                   int k) {
  // k = bank: the predictor-gated dense FFN (every channel kept), no ranking
  if (k >= bank) return bank >= 64 ? ~0ull : ((1ull << bank) - 1ull);
  const int lane = threadIdx.x & 31;
  int r0 = 0, r1 = 0;
#pragma unroll 8
  for (int j = 0; j < 32; ++j) {
    const uint32_t a = __shfl_sync(kFull, key0, j);  // channel j
    const uint32_t c = __shfl_sync(kFull, key1, j);  // channel j + 32
    if (j < bank) {
      r0 += (a > key0) | ((a == key0) & (j < lane));
      r1 += (a >= key1);  // channel j < lane + 32 always: ties go to j
    }
    if (j + 32 < bank) {
      r0 += (c > key0);  // channel j + 32 > lane: ties stay with lane
      r1 += (c > key1) | ((c == key1) & (j < lane));
    }
  }
  const bool s0 = (lane < bank) && (r0 < k);
  const bool s1 = (lane + 32 < bank) && (r1 < k);
  const uint32_t lo = __ballot_sync(kFull, s0);
  const uint32_t hi = __ballot_sync(kFull, s1);
  return ((uint64_t)hi << 32) | lo;
}

// Descending compare-exchange on order keys.
__device__ __forceinline__ void cex_desc(uint32_t &a, uint32_t &b) {
  const uint32_t hi = max(a, b), lo = min(a, b);
  a = hi;
  b = lo;
}

// Bitonic network sorting s[OFF, OFF + N) of an array of any length in
// descending order.  Every index is a compile-time constant (the stages are
// template-recursive), so the array stays in registers.
template <int OFF, int N, int SIZE, int STRIDE>
struct BitonicStage {
  template <int L>
  __device__ __forceinline__ static void run(uint32_t (&s)[L]) {
    static_assert(OFF + N <= L, "network outside the array");
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int j = i ^ STRIDE;
      if (j > i) {
        if ((i & SIZE) == 0)
          cex_desc(s[OFF + i], s[OFF + j]);
        else
          cex_desc(s[OFF + j], s[OFF + i]);
      }
    }
    BitonicStage<OFF, N, SIZE, STRIDE / 2>::run(s);
  }
};
template <int OFF, int N, int SIZE>
struct BitonicStage<OFF, N, SIZE, 0> {
  template <int L>
  __device__ __forceinline__ static void run(uint32_t (&)[L]) {}
};
template <int OFF, int N, int SIZE>
struct BitonicSort {
  template <int L>
  __device__ __forceinline__ static void run(uint32_t (&s)[L]) {
    BitonicStage<OFF, N, SIZE, SIZE / 2>::run(s);
    BitonicSort<OFF, N, SIZE * 2>::run(s);
  }
};
template <int OFF, int N>
struct BitonicSort<OFF, N, 2 * N> {
  template <int L>
  __device__ __forceinline__ static void run(uint32_t (&)[L]) {}
};

// Warp sums of four per-lane values in six shuffles (four separate
// reductions take twenty, each a chain of dependent shuffles).  On return the
// eight lanes with bits 4, 3 of the lane index equal to (a, b) hold the sum of
// value 2a + b.
__device__ __forceinline__ float warp_sum4(float v0, float v1, float v2, float v3) {
  const int lane = threadIdx.x & 31;
  const bool hi16 = (lane & 16) != 0, hi8 = (lane & 8) != 0;
  float s0 = hi16 ? v2 : v0, s1 = hi16 ? v3 : v1;
  s0 += __shfl_xor_sync(kFull, hi16 ? v0 : v2, 16);
  s1 += __shfl_xor_sync(kFull, hi16 ? v1 : v3, 16);
  float r = hi8 ? s1 : s0;
  r += __shfl_xor_sync(kFull, hi8 ? s0 : s1, 8);
  r += __shfl_xor_sync(kFull, r, 4);
  r += __shfl_xor_sync(kFull, r, 2);
  r += __shfl_xor_sync(kFull, r, 1);
  return r;
}

// The same top-k, for a bank whose order keys are in shared memory (keys[j],
// j < bank; the array padded to 64 entries with any values, 16-byte aligned),
// by one warp: every lane reads all keys with broadcast loads and counts the
// ranks of its two channels itself.  A chain of warp shuffles is latency
// bound; this has no cross-lane dependency until the two ballots.
__device__ __forceinline__ uint64_t smem_bank_topk(const uint32_t *keys, int bank, int k) {
  if (k >= bank) return bank >= 64 ? ~0ull : ((1ull << bank) - 1ull);
  const int lane = threadIdx.x & 31;
  const uint32_t key0 = keys[lane], key1 = keys[lane + 32];
  int r0 = 0, r1 = 0;
#pragma unroll 4
  for (int j0 = 0; j0 < 64; j0 += 4) {
    const uint4 q = *reinterpret_cast<const uint4 *>(keys + j0);
    const uint32_t kj[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + e;
      const bool in = j < bank;
      r0 += in & ((kj[e] > key0) | ((kj[e] == key0) & (j < lane)));
      r1 += in & ((kj[e] > key1) | ((kj[e] == key1) & (j < lane + 32)));
    }
  }
  const bool s0 = (lane < bank) && (r0 < k);
  const bool s1 = (lane + 32 < bank) && (r1 < k);
  const uint32_t lo = __ballot_sync(kFull, s0);
  const uint32_t hi = __ballot_sync(kFull, s1);
  return ((uint64_t)hi << 32) | lo;
}

// --------------------------------------------------------------- host side
struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int max_smem_optin = 0;
  unsigned *err = nullptr;  // device address of the library's error word
};
// Cached per-device properties; returns false if no device is usable.
bool device_info(DeviceInfo *out);

void count_launches(uint64_t n);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, once per (kernel, device, size class); no-op up to 48 KB.
// Done before the first launch so that no attribute call happens later, for
// example inside a stream capture.
cudaError_t ensure_smem_limit(const void *kernel, size_t bytes);

// Shape of one forward call, after validation.
struct FwdShape {
  int64_t T;
  int d, d_i, r, bank, k;
  int n_banks, d_s;
  bool bf16;
};

// Scratch carve-up of the CUDA-core (gather) path.
struct GatherPlan {
  int tt_h;  // tokens per CTA of the h kernel
  int tt_p;  // tokens per CTA of the logits/top-k kernel
  int cpt;   // CTAs per token of the gate/up/down kernel
  size_t off_h, off_idx, off_sig, off_part, total;
};
GatherPlan plan_gather(const FwdShape &s);
int pred_tokens_per_cta(const FwdShape &s);

// Launch with programmatic stream serialisation (programmatic dependent
// launch): the kernel may start while its predecessor in the stream is still
// running and must call griddepcontrol.wait before touching its outputs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Launchers (enqueue only; return the launch status).
// prefetch (may be null): prefetch_bytes of weights (a multiple of 16) that
// the next kernel reads, brought into L2 in the h kernel's prologue.
cudaError_t launch_pred_h(const FwdShape &s, int tt, const void *x, const void *A, void *h,
                          bool split_out, cudaStream_t st, const void *prefetch = nullptr,
                          size_t prefetch_bytes = 0);
cudaError_t launch_logits_topk(const FwdShape &s, int tt, const float *h, const void *B,
                               float *logits, uint64_t *mask, int *sel_idx, float *sel_sig,
                               unsigned *err, cudaStream_t st);
cudaError_t launch_bank_topk(const float *logits, uint64_t *mask, int64_t T, int d_i,
                             int bank, int k, cudaStream_t st);

bool ffn_shape_ok(const FwdShape &s);
int ffn_ctas_per_token(const FwdShape &s, int num_sms);
cudaError_t launch_ffn(const FwdShape &s, int cpt, const void *x, const int *sel_idx,
                       const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                       float *partial, unsigned *err, cudaStream_t st);
// Output of k_reduce_partials: y in the call's element type, or the bf16
// hi/lo halves of h ([T][2r], "split").
// kYF32: y as float32 whatever the input type (partial outputs of a bank
// shard, summed across devices before rounding).
enum class ReduceOut { kY, kYF32, kSplitH };

cudaError_t launch_reduce_partials(const FwdShape &s, int cpt, const float *partial, void *y,
                                   cudaStream_t st, ReduceOut kind = ReduceOut::kY);

// ---------------------------------------------------------------- backward
cudaError_t launch_bank_tau(const float *logits, uint64_t *mask, float *tau, int64_t T, int d_i,
                            int bank, int k, cudaStream_t st);
cudaError_t launch_bwd_elem(const float *P, const uint64_t *mask, const float *tau,
                            const float *G, const float *U, const float *DA, uint16_t *a,
                            uint16_t *dg, uint16_t *du, uint16_t *dp, int64_t T, int d_i,
                            int bank, float temp, cudaStream_t st);
cudaError_t launch_f32_to_bf16(const float *in, uint16_t *out, int64_t n, cudaStream_t st);

// Scratch carve-up of the tensor-core path.
struct TcPlan {
  int ksplit;  // K ranges of the down GEMM (fp32 partials reduced after)
  int hsplit;  // K ranges of the h GEMM (fp32 partials reduced + split after)
  size_t off_h2, off_sig, off_act, off_mask, off_part, off_hpart, total;
};
int tc_down_splits(const FwdShape &s, int num_sms);
int tc_h_splits(const FwdShape &s, int num_sms);
bool tc_shape_ok(const FwdShape &s);
TcPlan plan_tc(const FwdShape &s);
cudaError_t launch_tc_h(const FwdShape &s, const DeviceInfo &dev, const void *x, const void *A,
                        uint16_t *h2, float *partial, int ksplit, cudaStream_t st);
cudaError_t launch_tc_logits(const FwdShape &s, const DeviceInfo &dev, const uint16_t *h2,
                             const void *B, float *logits, uint64_t *mask, float *sig,
                             cudaStream_t st);
cudaError_t launch_tc_gateup(const FwdShape &s, const DeviceInfo &dev, const void *x,
                             const void *Wg, const void *Wu, const uint64_t *mask,
                             const float *sig, uint16_t *act, cudaStream_t st);
// With all tokens in one 128-row tile: the logits GEMM, the bank top-k and
// the masked gate/up in one kernel (mask may be null).
bool tc_fused_gateup_ok(const FwdShape &s);
cudaError_t launch_tc_logits_gateup(const FwdShape &s, const DeviceInfo &dev,
                                    const uint16_t *h2, const void *B, const void *x,
                                    const void *Wg, const void *Wu, uint64_t *mask,
                                    uint16_t *act, cudaStream_t st);
cudaError_t launch_tc_dense4x_gateup(const FwdShape &s, const DeviceInfo &dev, const void *x,
                                     const void *Wg, const void *Wu, uint64_t *mask,
                                     uint16_t *act, cudaStream_t st);
cudaError_t launch_tc_logits_tau(const FwdShape &s, const DeviceInfo &dev, const uint16_t *h2,
                                 const void *B, float *logits, uint64_t *mask, float *tau,
                                 cudaStream_t st);
cudaError_t launch_tc_down(const FwdShape &s, const DeviceInfo &dev, const uint16_t *act,
                           const void *Wd, void *y, int ksplit, cudaStream_t st,
                           bool f32_out = false);
// C[M][ldc] (=, or += when accumulate) A B on the tensor cores: bf16
// operands, float32 out.  A [M][K] (row stride lda), or [K][M] when a_mn; B
// [N][K] (ldb), or [K][N] when b_mn.  N % 64 == 0; a_mn needs b_mn.
cudaError_t launch_tc_gemm_f32(const DeviceInfo &dev, int M, int N, int K, const void *A,
                               int lda, bool a_mn, const void *B, int ldb, bool b_mn, float *C,
                               int ldc, bool accumulate, cudaStream_t st);

}  // namespace sfn
