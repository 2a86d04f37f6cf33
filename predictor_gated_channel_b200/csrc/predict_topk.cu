// predict_topk.cu -- CUDA-core kernels of the predictor and the bank top-k
// (the few-token path, and the standalone top-k).
//
// Predictor "R^d -> R^448 -> R^{d_i}" and the bank-wise hard top-16 of 64:
// "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity Training
// Recipe for Dense-to-Sparse LLMs", gist.science summary, "1. Architectuur".
//
//   k_pred_h       h[t] = A x[t] (fp32), one warp per row of A with the whole
//                  row's 16-byte loads in flight; token groups of TT share
//                  each row load.  The first token group also issues L2
//                  prefetches of B, so that k_logits_topk reads B from L2.
//   k_logits_topk  p[t] = B h[t] for one bank, then (optionally) that bank's
//                  top-k: mask word, kept channel ids and sigma(p) in
//                  ascending channel order (one CTA per bank and token group)
//   k_bank_topk    standalone top-k on float32 logits (one warp per bank)
//
// Both chained kernels use programmatic dependent launch: they let the next
// kernel start early, issue only L2 prefetches of weights before
// griddepcontrol.wait, and touch every other buffer after it.
#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Stage TT token rows of x (element type E) into shared memory as float;
// rows past the end of the batch are zero.
template <class E, int TT>
__device__ __forceinline__ void stage_rows(float *xs, const char *x, int64_t t0, int nt,
                                           int d) {
  const int nchunk = d / E::kVec;
  for (int i = threadIdx.x; i < TT * nchunk; i += blockDim.x) {
    const int t = i / nchunk, c = i - t * nchunk;
    float f[E::kVec];
    if (t < nt) {
      const uint4 v = ld_nc16(x + ((t0 + t) * (int64_t)d + (int64_t)c * E::kVec) * E::kBytes);
      E::unpack(v, f);
    } else {
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) f[e] = 0.f;
    }
    float4 *dst = reinterpret_cast<float4 *>(xs + t * d + c * E::kVec);
#pragma unroll
    for (int e = 0; e < E::kVec / 4; ++e)
      dst[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
  }
}

// h[t][m] = sum_n A[m][n] x[t][n].  1-D grid over (token group, row block):
// blockIdx.x = token_group * ceil(r / kWarps) + row_block.
// If Bpf != nullptr, the CTAs of token group 0 prefetch B (Bpf_bytes) to L2.
template <class E, int TT>
__global__ void __launch_bounds__(kThreads) k_pred_h(const char *__restrict__ x,
                                                     const char *__restrict__ A,
                                                     float *__restrict__ h, int64_t T, int d,
                                                     int r, const char *__restrict__ Bpf,
                                                     int64_t Bpf_bytes) {
  extern __shared__ float4 smem_f4[];
  float *xs = reinterpret_cast<float *>(smem_f4);
  const int row_blocks = (r + kWarps - 1) / kWarps;
  const int64_t tg = blockIdx.x / row_blocks;
  const int rb = blockIdx.x % row_blocks;
  pdl_launch_dependents();
  if (Bpf != nullptr && tg == 0 && threadIdx.x == 0) {
    // this CTA's 16-byte-aligned share of B
    const int64_t share = ((Bpf_bytes + row_blocks - 1) / row_blocks + 15) / 16 * 16;
    const int64_t beg = rb * share;
    const int64_t end = beg + share < Bpf_bytes ? beg + share : Bpf_bytes;
    for (int64_t o = beg; o < end; o += 65536) {
      const int64_t n = end - o < 65536 ? end - o : 65536;
      prefetch_l2(Bpf + o, (uint32_t)n);
    }
  }
  pdl_wait();

  const int64_t t0 = tg * TT;
  const int nt = (T - t0 < TT) ? (int)(T - t0) : TT;
  stage_rows<E, TT>(xs, x, t0, nt, d);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = rb * kWarps + warp;
  if (m >= r) return;
  const int nchunk = d / E::kVec;
  const char *row = A + (int64_t)m * d * E::kBytes;
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  // 16 loads per lane in flight (a whole 8 KB bf16 row per warp)
  for (int c0 = lane; c0 < nchunk; c0 += 32 * 16) {
    uint4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = c0 + 32 * u;
      v[u] = (c < nchunk) ? ld_stream16(row + (int64_t)c * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        float a[E::kVec];
        E::unpack(v[u], a);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          const float *xr = xs + t * d + c * E::kVec;
#pragma unroll
          for (int e = 0; e < E::kVec; ++e) acc[t] = fmaf(a[e], xr[e], acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const float v = warp_sum(acc[t]);
    if (lane == 0 && t < nt) h[(t0 + t) * r + m] = v;
  }
}

// Logits of one bank for TT tokens, then the bank's top-k.  1-D grid:
// blockIdx.x = token_group * n_banks + bank_index.
//   logits  : if kWriteLogits, [T][d_i] float32
//   mask    : if non-null, [T][n_banks] uint64
//   sel_idx : if kTopk, [T][d_s] channel ids of kept channels, bank-major,
//             ascending inside each bank; sel_sig the matching sigma(p)
template <class E, int TT, bool kWriteLogits, bool kTopk>
__global__ void __launch_bounds__(kThreads) k_logits_topk(
    const float *__restrict__ h, const char *__restrict__ B, float *__restrict__ logits,
    uint64_t *__restrict__ mask, int *__restrict__ sel_idx, float *__restrict__ sel_sig,
    int64_t T, int d_i, int r, int bank, int k) {
  extern __shared__ float4 smem_f4[];
  float *hs = reinterpret_cast<float *>(smem_f4);  // [TT][r]
  float *ps = hs + TT * r;                         // [TT][64]
  const int n_banks = d_i / bank;
  const int b = blockIdx.x % n_banks;
  const int64_t t0 = (int64_t)(blockIdx.x / n_banks) * TT;
  const int nt = (T - t0 < TT) ? (int)(T - t0) : TT;
  pdl_launch_dependents();
  pdl_wait();
  for (int i = threadIdx.x; i < TT * r; i += blockDim.x) {
    const int t = i / r;
    hs[i] = (t < nt) ? h[(t0 + t) * r + (i - t * r)] : 0.f;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = r / E::kVec;
  // Each warp owns rows jl = warp + kWarps * i; a group of 4 rows x 2 chunk
  // columns of loads is issued before any arithmetic.
  for (int jl0 = warp; jl0 < bank; jl0 += 4 * kWarps) {
    float acc[4][TT];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[q][t] = 0.f;
    for (int c0 = lane; c0 < nchunk; c0 += 64) {
      uint4 v[4][2];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int jl = jl0 + q * kWarps;
        const char *row = B + (int64_t)(b * bank + jl) * r * E::kBytes;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + 32 * u;
          v[q][u] = (jl < bank && c < nchunk) ? ld_nc16(row + (int64_t)c * 16)
                                              : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + 32 * u;
          if (c < nchunk) {
            float w[E::kVec];
            E::unpack(v[q][u], w);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              const float *hr = hs + t * r + c * E::kVec;
#pragma unroll
              for (int e = 0; e < E::kVec; ++e) acc[q][t] = fmaf(w[e], hr[e], acc[q][t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int jl = jl0 + q * kWarps;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float v = warp_sum(acc[q][t]);
        if (lane == 0 && jl < bank) {
          ps[t * 64 + jl] = v;
          if (kWriteLogits && t < nt) logits[(t0 + t) * d_i + b * bank + jl] = v;
        }
      }
    }
  }
  if (!kTopk) return;
  __syncthreads();

  const int d_s = n_banks * k;
  for (int t = warp; t < nt; t += kWarps) {
    const float p0 = (lane < bank) ? ps[t * 64 + lane] : 0.f;
    const float p1 = (lane + 32 < bank) ? ps[t * 64 + lane + 32] : 0.f;
    const uint64_t word = warp_bank_topk(order_key(p0), order_key(p1), bank, k);
    const int64_t tg = t0 + t;
    if (mask != nullptr && lane == 0) mask[tg * n_banks + b] = word;
    int *idx_row = sel_idx + tg * d_s + b * k;
    float *sig_row = sel_sig + tg * d_s + b * k;
    if ((word >> lane) & 1ull) {
      const int s = __popcll(word & ((1ull << lane) - 1ull));
      idx_row[s] = b * bank + lane;
      sig_row[s] = sigmoid_f32(p0);
    }
    if ((word >> (lane + 32)) & 1ull) {
      const int s = __popcll(word & ((1ull << (lane + 32)) - 1ull));
      idx_row[s] = b * bank + lane + 32;
      sig_row[s] = sigmoid_f32(p1);
    }
  }
}

// Standalone top-k: one warp per (token, bank).
__global__ void __launch_bounds__(kThreads) k_bank_topk(const float *__restrict__ logits,
                                                        uint64_t *__restrict__ mask,
                                                        int64_t n_words, int bank, int k) {
  const int64_t wi = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (wi >= n_words) return;  // whole warp leaves together
  const int lane = threadIdx.x & 31;
  const float *p = logits + wi * bank;  // banks of a row are contiguous
  const uint32_t k0 = (lane < bank) ? order_key(p[lane]) : 0u;
  const uint32_t k1 = (lane + 32 < bank) ? order_key(p[lane + 32]) : 0u;
  const uint64_t word = warp_bank_topk(k0, k1, bank, k);
  if (lane == 0) mask[wi] = word;
}

template <class E, int TT>
cudaError_t pred_h_tt(const FwdShape &s, const void *x, const void *A, float *h,
                      const void *Bpf, cudaStream_t st) {
  const size_t smem = (size_t)TT * s.d * sizeof(float);
  auto kern = k_pred_h<E, TT>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)((s.r + kWarps - 1) / kWarps) * ((s.T + TT - 1) / TT);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int64_t bpf_bytes = (int64_t)s.d_i * s.r * (s.bf16 ? 2 : 4);
  e = launch_pdl(kern, dim3((unsigned)blocks), dim3(kThreads), smem, st, (const char *)x,
                 (const char *)A, h, s.T, s.d, s.r, (const char *)Bpf, bpf_bytes);
  count_launches(1);
  return e;
}

template <class E, int TT, bool W, bool K>
cudaError_t logits_tt(const FwdShape &s, const float *h, const void *B, float *logits,
                      uint64_t *mask, int *sel_idx, float *sel_sig, cudaStream_t st) {
  const size_t smem = (size_t)TT * (s.r + 64) * sizeof(float);
  auto kern = k_logits_topk<E, TT, W, K>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)s.n_banks * ((s.T + TT - 1) / TT);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  e = launch_pdl(kern, dim3((unsigned)blocks), dim3(kThreads), smem, st, h, (const char *)B,
                 logits, mask, sel_idx, sel_sig, s.T, s.d_i, s.r, s.bank, s.k);
  count_launches(1);
  return e;
}

template <class E, bool W, bool K>
cudaError_t logits_dispatch(const FwdShape &s, int tt, const float *h, const void *B,
                            float *logits, uint64_t *mask, int *sel_idx, float *sel_sig,
                            cudaStream_t st) {
  switch (tt) {
    case 1: return logits_tt<E, 1, W, K>(s, h, B, logits, mask, sel_idx, sel_sig, st);
    case 2: return logits_tt<E, 2, W, K>(s, h, B, logits, mask, sel_idx, sel_sig, st);
    case 4: return logits_tt<E, 4, W, K>(s, h, B, logits, mask, sel_idx, sel_sig, st);
    default: return logits_tt<E, 8, W, K>(s, h, B, logits, mask, sel_idx, sel_sig, st);
  }
}

}  // namespace

cudaError_t launch_pred_h(const FwdShape &s, int tt, const void *x, const void *A, float *h,
                          const void *Bpf, cudaStream_t st) {
  if (s.bf16) {
    switch (tt) {
      case 1: return pred_h_tt<EltBF16, 1>(s, x, A, h, Bpf, st);
      case 2: return pred_h_tt<EltBF16, 2>(s, x, A, h, Bpf, st);
      case 4: return pred_h_tt<EltBF16, 4>(s, x, A, h, Bpf, st);
      default: return pred_h_tt<EltBF16, 8>(s, x, A, h, Bpf, st);
    }
  }
  switch (tt) {
    case 1: return pred_h_tt<EltF32, 1>(s, x, A, h, Bpf, st);
    case 2: return pred_h_tt<EltF32, 2>(s, x, A, h, Bpf, st);
    case 4: return pred_h_tt<EltF32, 4>(s, x, A, h, Bpf, st);
    default: return pred_h_tt<EltF32, 8>(s, x, A, h, Bpf, st);
  }
}

cudaError_t launch_logits_topk(const FwdShape &s, int tt, const float *h, const void *B,
                               float *logits, uint64_t *mask, int *sel_idx, float *sel_sig,
                               cudaStream_t st) {
  const bool topk = sel_idx != nullptr;
  const bool write = logits != nullptr;
  if (s.bf16) {
    if (topk && write)
      return logits_dispatch<EltBF16, true, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
    if (topk)
      return logits_dispatch<EltBF16, false, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
    return logits_dispatch<EltBF16, true, false>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
  }
  if (topk && write)
    return logits_dispatch<EltF32, true, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
  if (topk)
    return logits_dispatch<EltF32, false, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
  return logits_dispatch<EltF32, true, false>(s, tt, h, B, logits, mask, sel_idx, sel_sig, st);
}

cudaError_t launch_bank_topk(const float *logits, uint64_t *mask, int64_t T, int d_i,
                             int bank, int k, cudaStream_t st) {
  const int64_t n_words = T * (d_i / bank);
  const int64_t blocks = (n_words + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  k_bank_topk<<<(unsigned)blocks, kThreads, 0, st>>>(logits, mask, n_words, bank, k);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace sfn
