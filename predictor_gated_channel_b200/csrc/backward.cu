// backward.cu -- the layer's backward pass for predictor training, with the
// soft surrogate gradient of the bank top-k.
//
// "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity Training
// Recipe for Dense-to-Sparse LLMs", gist.science summary, "1. Architectuur",
// Executie / Backward Pass: the hard top-k is not differentiable; a soft,
// sigmoid-like surrogate gradient around the selection threshold lets the
// loss reach the predictor.  Reading (the pages give no formula): bank b's
// threshold tau_b is the midpoint of its k-th and (k+1)-th logits, held
// constant, and dm_j/dp_j := sigma'((p_j - tau_b) / temp) / temp.
//
//   k_bank_tau    per (token, bank), one thread: the hard top-k mask (the
//                 forward's rule) and tau_b (NaN when k = bank: no threshold,
//                 no surrogate), from a register sorting network
//   k_bwd_elem    per (token, channel), from the logits p, the mask, tau and
//                 g = Wg x, u = Wu x, da = Wd dy (float32):
//                   a  = m s g u                      (s = sigma(p))
//                   dg = da m s u,  du = da m s g,
//                   dp = da g u (m s (1 - s) + s sigma'(z) / temp)
//                 written as bf16 GEMM operands
//   k_f32_to_bf16 float32 -> bf16 rows (h and dh as GEMM operands)
//
// The dense contractions around them (g, u, da; the weight gradients; dh,
// dx) run on the library's tcgen05 GEMM (tc_path.cu, launch_tc_gemm_f32:
// bf16 operands, float32 accumulation and output).
#include <cmath>

#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kElemThreads = 256;
constexpr int kTauThreads = 128;

// One thread per (token, bank): the bank's logits become order keys (padding
// past `bank` gets key 0, below every number), a register bitonic network
// sorts a copy, the k-th and (k+1)-th keys give the threshold, and the mask
// takes every key above the k-th plus, in channel order, as many equal to it
// as are still needed (equal logits to the lower index).
__global__ void __launch_bounds__(kTauThreads) k_bank_tau(const float *__restrict__ logits,
                                                          uint64_t *__restrict__ mask,
                                                          float *__restrict__ tau,
                                                          int64_t n_words, int bank, int k) {
  // The block's banks are one contiguous run of logits (the banks of a token
  // row are contiguous): read it coalesced into rows of bank + 1 floats, so
  // that the threads' reads of their own rows hit distinct smem banks.
  __shared__ float tile[kTauThreads * 65];
  const int64_t w0 = (int64_t)blockIdx.x * kTauThreads;
  const int nw = (int)((n_words - w0 < kTauThreads) ? n_words - w0 : kTauThreads);
  const float *src = logits + w0 * bank;
  const int total = nw * bank;
  for (int f0 = threadIdx.x; f0 < total; f0 += 16 * kTauThreads) {
    float v[16];  // 16 loads in flight per thread before any store
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int f = f0 + u * kTauThreads;
      v[u] = (f < total) ? src[f] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int f = f0 + u * kTauThreads;
      if (f < total) {
        const int row = f / bank;
        tile[row * (bank + 1) + (f - row * bank)] = v[u];
      }
    }
  }
  __syncthreads();
  if ((int)threadIdx.x >= nw) return;
  const int64_t wi = w0 + threadIdx.x;
  const float *p = tile + threadIdx.x * (bank + 1);
  uint32_t key[64], s[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    key[i] = (i < bank) ? order_key(p[i]) : 0u;
    s[i] = key[i];
  }
  BitonicSort<0, 64, 2>::run(s);
  uint32_t kth = s[0], next = 0u;
#pragma unroll
  for (int i = 1; i < 64; ++i) {
    kth = (i == k - 1) ? s[i] : kth;
    next = (i == k) ? s[i] : next;
  }
  int gt = 0;
#pragma unroll
  for (int i = 0; i < 64; ++i) gt += key[i] > kth;
  const int need = k - gt;
  int eq = 0;
  uint64_t word = 0;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const bool take = (i < bank) & ((key[i] > kth) | ((key[i] == kth) & (eq < need)));
    eq += (i < bank) & (key[i] == kth);
    word |= (uint64_t)take << i;
  }
  if (mask != nullptr) mask[wi] = word;
  tau[wi] = (k < bank) ? 0.5f * (key_value(kth) + key_value(next)) : __int_as_float(0x7fc00000);
}

__device__ __forceinline__ float sigmoid_acc(float z) { return 1.0f / (1.0f + expf(-z)); }

// Elementwise chain rule of the layer, 4 channels per thread (d_i % 4 == 0,
// so the 4 share one token).
__global__ void __launch_bounds__(kElemThreads) k_bwd_elem(
    const float *__restrict__ P, const uint64_t *__restrict__ mask, const float *__restrict__ tau,
    const float *__restrict__ G, const float *__restrict__ U, const float *__restrict__ DA,
    uint16_t *__restrict__ a_out, uint16_t *__restrict__ dg_out, uint16_t *__restrict__ du_out,
    uint16_t *__restrict__ dp_out, int64_t n4, int d_i, int bank, float inv_temp) {
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= n4) return;
  const int64_t e0 = q * 4;
  const int64_t t = e0 / d_i;
  const int j0 = (int)(e0 - t * d_i);
  const int nb = d_i / bank;
  const float4 p4 = *reinterpret_cast<const float4 *>(P + e0);
  const float4 g4 = *reinterpret_cast<const float4 *>(G + e0);
  const float4 u4 = *reinterpret_cast<const float4 *>(U + e0);
  const float4 d4 = *reinterpret_cast<const float4 *>(DA + e0);
  const float pv[4] = {p4.x, p4.y, p4.z, p4.w}, gv[4] = {g4.x, g4.y, g4.z, g4.w};
  const float uv[4] = {u4.x, u4.y, u4.z, u4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
  uint16_t ao[4], go[4], uo[4], po[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = (j0 + e) / bank;
    const float tb = tau[t * nb + b];
    const float m = (float)((mask[t * nb + b] >> ((j0 + e) - b * bank)) & 1ull);
    const float s = sigmoid_acc(pv[e]);
    float sur = 0.f;
    if (!isnan(tb)) {
      const float sz = sigmoid_acc((pv[e] - tb) * inv_temp);
      sur = sz * (1.f - sz) * inv_temp;
    }
    const float gu = gv[e] * uv[e];
    ao[e] = f32_to_bf16_bits(m * s * gu);
    go[e] = f32_to_bf16_bits(dv[e] * m * s * uv[e]);
    uo[e] = f32_to_bf16_bits(dv[e] * m * s * gv[e]);
    po[e] = f32_to_bf16_bits(dv[e] * gu * (m * s * (1.f - s) + s * sur));
  }
  auto pack = [](const uint16_t *v) {
    return make_uint2((uint32_t)v[0] | ((uint32_t)v[1] << 16),
                      (uint32_t)v[2] | ((uint32_t)v[3] << 16));
  };
  *reinterpret_cast<uint2 *>(a_out + e0) = pack(ao);
  *reinterpret_cast<uint2 *>(dg_out + e0) = pack(go);
  *reinterpret_cast<uint2 *>(du_out + e0) = pack(uo);
  *reinterpret_cast<uint2 *>(dp_out + e0) = pack(po);
}

__global__ void __launch_bounds__(kElemThreads) k_f32_to_bf16(const float *__restrict__ in,
                                                              uint16_t *__restrict__ out,
                                                              int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = f32_to_bf16_bits(in[i]);
}

}  // namespace

cudaError_t launch_bank_tau(const float *logits, uint64_t *mask, float *tau, int64_t T, int d_i,
                            int bank, int k, cudaStream_t st) {
  const int64_t n_words = T * (d_i / bank);
  const int64_t blocks = (n_words + kTauThreads - 1) / kTauThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  k_bank_tau<<<(unsigned)blocks, kTauThreads, 0, st>>>(logits, mask, tau, n_words, bank, k);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_elem(const float *P, const uint64_t *mask, const float *tau,
                            const float *G, const float *U, const float *DA, uint16_t *a,
                            uint16_t *dg, uint16_t *du, uint16_t *dp, int64_t T, int d_i,
                            int bank, float temp, cudaStream_t st) {
  const int64_t n4 = T * (int64_t)d_i / 4;
  const int64_t blocks = (n4 + kElemThreads - 1) / kElemThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  k_bwd_elem<<<(unsigned)blocks, kElemThreads, 0, st>>>(P, mask, tau, G, U, DA, a, dg, du, dp,
                                                       n4, d_i, bank, 1.0f / temp);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float *in, uint16_t *out, int64_t n, cudaStream_t st) {
  const int64_t blocks = (n + kElemThreads - 1) / kElemThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (n == 0) return cudaSuccess;
  k_f32_to_bf16<<<(unsigned)blocks, kElemThreads, 0, st>>>(in, out, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace sfn
