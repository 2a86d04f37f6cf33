// predict_topk.cu -- CUDA-core kernels of the predictor and the bank top-k
// (the few-token path, and the standalone top-k).
//
// The predictor, a two-layer map R^d -> R^448 -> R^{d_i}, and the bank-wise
// hard top-16 of 64:
// "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity Training
// Recipe for Dense-to-Sparse LLMs", gist.science summary, "1. Architectuur".
//
//   k_pred_h       h[t] = A x[t] (fp32), one warp per row of A with the whole
//                  row's 16-byte loads in flight; token groups of TT share
//                  each row load.  x's lines are L2-prefetched before the
//                  wait; one token's x then goes straight into registers.
//   k_logits_topk  p[t] = B h[t] for one bank, then (optionally) that bank's
//                  top-k: mask word, kept channel ids and sigma(p) in
//                  ascending channel order (one CTA per bank and token group).
//                  The bank's block of B (64 contiguous rows) is bulk-copied
//                  into shared memory in the prologue, while k_pred_h runs.
//   k_bank_topk    standalone top-k on float32 logits (one warp per bank)
//
// The chained kernels use programmatic dependent launch.  Each calls
// griddepcontrol.wait before touching anything an earlier kernel writes and
// only then lets its dependent start, so a dependent's prologue (which reads
// nothing but weights; the L2 prefetch of x is a hint, not a read of its
// values) always runs after all work before its predecessor.
#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kThreadsH = 128;          // k_pred_h: 4 rows of A per CTA
constexpr int kWarpsH = kThreadsH / 32;
constexpr uint32_t kMaxBBlock = 96 * 1024;  // bank block of B staged in smem

// Stage TT token rows of x (element type E) into shared memory as float;
// rows past the end of the batch are zero.  Each thread issues up to 8 of its
// loads before any store, so a row costs one memory round trip.
template <class E, int TT>
__device__ __forceinline__ void stage_rows(float *xs, const char *x, int64_t t0, int nt,
                                           int d) {
  const int nchunk = d / E::kVec;
  const int total = TT * nchunk;
  for (int i0 = threadIdx.x; i0 < total; i0 += 8 * blockDim.x) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      const int t = i / nchunk, c = i - t * nchunk;
      v[u] = (i < total && t < nt)
                 ? ld_nc16(x + ((t0 + t) * (int64_t)d + (int64_t)c * E::kVec) * E::kBytes)
                 : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < total) {
        float f[E::kVec];
        E::unpack(v[u], f);
        float4 *dst = reinterpret_cast<float4 *>(xs + (size_t)i * E::kVec);
#pragma unroll
        for (int e = 0; e < E::kVec / 4; ++e)
          dst[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
      }
    }
  }
}

// h[t][m] = sum_n A[m][n] x[t][n].  1-D grid over (token group, row block):
// blockIdx.x = token_group * ceil(r / kWarpsH) + row_block.
// kSplitOut: instead of fp32 h [T][r], write h as two bf16 halves
// hi = bf16(h), lo = bf16(h - hi) into [T][2r] (hi first), the operand form
// of the tensor-core logits GEMM.
// pf (may be null): pf_bytes of weights the next kernel reads (the rows of
// B), prefetched into L2 by the first token group's CTAs in the prologue,
// together with this CTA's rows of A, before griddepcontrol.wait.
template <class E, int TT, bool kSplitOut>
__global__ void __launch_bounds__(kThreadsH) k_pred_h(const char *__restrict__ x,
                                                      const char *__restrict__ A,
                                                      void *__restrict__ h_out, int64_t T,
                                                      int d, int r, const char *__restrict__ pf,
                                                      int64_t pf_bytes) {
  extern __shared__ float4 smem_f4[];
  float *xs = reinterpret_cast<float *>(smem_f4);
  const int row_blocks = (r + kWarpsH - 1) / kWarpsH;
  const int64_t tg = blockIdx.x / row_blocks;
  const int rb = blockIdx.x % row_blocks;
  if (pf != nullptr && tg == 0 && threadIdx.x < 32) {
    constexpr int64_t kPiece = 16384;
    const int64_t share = (pf_bytes / row_blocks + kPiece - 1) / kPiece * kPiece;
    const int64_t b0 = rb * share;
    const int64_t b1 = (b0 + share < pf_bytes) ? b0 + share : pf_bytes;
    for (int64_t o = b0 + threadIdx.x * kPiece; o < b1; o += 32 * kPiece)
      prefetch_l2(pf + o, (uint32_t)(b1 - o < kPiece ? b1 - o : kPiece));
  }

  const int64_t t0 = tg * TT;
  const int nt = (T - t0 < TT) ? (int)(T - t0) : TT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = rb * kWarpsH + warp;
  const int nchunk = d / E::kVec;
  const char *row = A + (int64_t)(m < r ? m : 0) * d * E::kBytes;
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  // The row's first 16 loads per lane go out before the wait and before x
  // is staged (8 KB bf16 rows: the whole row).
  uint4 v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int c = lane + 32 * u;
    v[u] = (m < r && c < nchunk) ? ld_stream16(row + (int64_t)c * 16) : make_uint4(0, 0, 0, 0);
  }
  // x's lines: warm before the wait (a hint; the loads below come after it)
  {
    const int64_t xb = (int64_t)nt * d * E::kBytes;
    const char *xr = x + t0 * (int64_t)d * E::kBytes;
    for (int64_t o = (int64_t)threadIdx.x * 128; o < xb; o += (int64_t)blockDim.x * 128)
      prefetch_line_l2(xr + o);
  }
  pdl_wait();  // x may come from earlier work on the stream
  pdl_launch_dependents();
  if (TT == 1 && nchunk <= 32 * 16) {
    // one token, the row in one pass: every lane loads the chunks of x that
    // match its chunks of A straight into registers (no staging, no barrier)
    if (m >= r) return;
    uint4 xv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = lane + 32 * u;
      xv[u] = (c < nchunk) ? ld_nc16(x + (t0 * (int64_t)d + (int64_t)c * E::kVec) * E::kBytes)
                           : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      float a[E::kVec], xf[E::kVec];
      E::unpack(v[u], a);
      E::unpack(xv[u], xf);
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) acc[0] = fmaf(a[e], xf[e], acc[0]);
    }
  } else {
  stage_rows<E, TT>(xs, x, t0, nt, d);
  __syncthreads();
  if (m >= r) return;
  for (int c0 = lane; c0 < nchunk; c0 += 32 * 16) {
    if (c0 != lane) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int c = c0 + 32 * u;
        v[u] = (c < nchunk) ? ld_stream16(row + (int64_t)c * 16) : make_uint4(0, 0, 0, 0);
      }
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
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const float v = warp_sum(acc[t]);
    if (lane == 0 && t < nt) {
      if (kSplitOut) {
        uint16_t *h2 = reinterpret_cast<uint16_t *>(h_out) + (t0 + t) * 2 * r;
        const uint16_t hi = f32_to_bf16_bits(v);
        h2[m] = hi;
        h2[r + m] = f32_to_bf16_bits(v - __uint_as_float((uint32_t)hi << 16));
      } else {
        reinterpret_cast<float *>(h_out)[(t0 + t) * r + m] = v;
      }
    }
  }
}

// Logits of one bank for TT tokens, then the bank's top-k.  1-D grid:
// blockIdx.x = token_group * n_banks + bank_index.
//   logits  : if kWriteLogits, [T][d_i] float32
//   mask    : if non-null, [T][n_banks] uint64
//   sel_idx : if kTopk, [T][d_s] channel ids of kept channels, bank-major,
//             ascending inside each bank; sel_sig the matching sigma(p)
// kSmemB: the bank's rows of B are staged in shared memory by bulk copies
// issued before griddepcontrol.wait (they are weights, not outputs of the
// previous kernel); otherwise they are read from global memory.
template <class E, int TT, bool kWriteLogits, bool kTopk, bool kSmemB>
__global__ void __launch_bounds__(kThreads) k_logits_topk(
    const float *__restrict__ h, const char *__restrict__ B, float *__restrict__ logits,
    uint64_t *__restrict__ mask, int *__restrict__ sel_idx, float *__restrict__ sel_sig,
    int64_t T, int d_i, int r, int bank, int k, unsigned *err) {
  extern __shared__ float4 smem_f4[];
  const uint32_t block_bytes = (uint32_t)bank * r * E::kBytes;
  unsigned char *bs = reinterpret_cast<unsigned char *>(smem_f4);      // [bank][r] (kSmemB)
  float *hs = reinterpret_cast<float *>(bs + (kSmemB ? block_bytes : 0));  // [TT][r]
  float *ps = hs + TT * r;                                              // [TT][64]
  uint32_t *pk = reinterpret_cast<uint32_t *>(ps + TT * 64);            // [TT][64] keys
  uint64_t *bbar = reinterpret_cast<uint64_t *>(pk + TT * 64);
  const int n_banks = d_i / bank;
  const int b = blockIdx.x % n_banks;
  const int64_t t0 = (int64_t)(blockIdx.x / n_banks) * TT;
  const int nt = (T - t0 < TT) ? (int)(T - t0) : TT;
  const char *bblock = B + (int64_t)b * block_bytes;
  if (kSmemB) {
    if (threadIdx.x == 0) {
      mbar_init(bbar, 1);
      fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(bbar, block_bytes);
      for (uint32_t o = 0; o < block_bytes; o += 16384) {
        const uint32_t n = block_bytes - o < 16384 ? block_bytes - o : 16384;
        bulk_g2s(bs + o, bblock + o, n, bbar);
      }
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  // h rows for the token group, float4 at a time (r % 4 == 0), all loads of
  // a thread issued before its stores
  for (int i0 = threadIdx.x; i0 < TT * r / 4; i0 += 4 * blockDim.x) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      const int t = 4 * i / r;
      v[u] = (i < TT * r / 4 && t < nt)
                 ? *reinterpret_cast<const float4 *>(h + (t0 + t) * r + (4 * i - t * r))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < TT * r / 4) reinterpret_cast<float4 *>(hs)[i] = v[u];
    }
  }
  __syncthreads();
  bool ok = true;
  if (kSmemB) {
    ok = __syncthreads_and(mbar_wait(bbar, 0, err)) != 0;
    // on a timeout, do not leave while the copies may still land
    if (!ok && threadIdx.x == 0) mbar_wait(bbar, 0, err);
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = r / E::kVec;
  // Each warp owns rows jl = warp + kWarps * i; a group of 4 rows x 2 chunk
  // columns of loads is issued before any arithmetic.
  for (int jl0 = warp; ok && jl0 < bank; jl0 += 4 * kWarps) {
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
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + 32 * u;
          const bool in = jl < bank && c < nchunk;
          if (kSmemB)
            v[q][u] = in ? *reinterpret_cast<const uint4 *>(bs + ((size_t)jl * r + (size_t)c * E::kVec) * E::kBytes)
                         : make_uint4(0, 0, 0, 0);
          else
            v[q][u] = in ? ld_nc16(bblock + ((int64_t)jl * r + (int64_t)c * E::kVec) * E::kBytes)
                         : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = c0 + 32 * u;
        if (c < nchunk) {
          // this chunk of h, for all tokens, read once and used for 4 rows
          float hv[TT][E::kVec];
#pragma unroll
          for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int e = 0; e < E::kVec; e += 4) {
              const float4 f = *reinterpret_cast<const float4 *>(hs + t * r + c * E::kVec + e);
              hv[t][e] = f.x;
              hv[t][e + 1] = f.y;
              hv[t][e + 2] = f.z;
              hv[t][e + 3] = f.w;
            }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float w[E::kVec];
            E::unpack(v[q][u], w);
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
              for (int e = 0; e < E::kVec; ++e) acc[q][t] = fmaf(w[e], hv[t][e], acc[q][t]);
          }
        }
      }
    }
    // the four rows' sums at once: lanes 8q .. 8q + 7 end with row q's
    const int q = lane >> 3;
    const int jl = jl0 + q * kWarps;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float v = warp_sum4(acc[0][t], acc[1][t], acc[2][t], acc[3][t]);
      if ((lane & 7) == 0 && jl < bank) {
        ps[t * 64 + jl] = v;
        pk[t * 64 + jl] = order_key(v);
        if (kWriteLogits && t < nt) logits[(t0 + t) * d_i + b * bank + jl] = v;
      }
    }
  }
  if (!kTopk || !ok) return;
  __syncthreads();

  const int d_s = n_banks * k;
  for (int t = warp; t < nt; t += kWarps) {
    const float p0 = (lane < bank) ? ps[t * 64 + lane] : 0.f;
    const float p1 = (lane + 32 < bank) ? ps[t * 64 + lane + 32] : 0.f;
    const uint64_t word = smem_bank_topk(pk + t * 64, bank, k);
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

template <class E, int TT, bool SPLIT>
cudaError_t pred_h_tt(const FwdShape &s, const void *x, const void *A, void *h,
                      const void *pf, size_t pf_bytes, cudaStream_t st) {
  // one token: x goes straight to registers, no staging
  const size_t smem = (TT == 1 && s.d / E::kVec <= 32 * 16) ? 0 : (size_t)TT * s.d * sizeof(float);
  auto kern = k_pred_h<E, TT, SPLIT>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)((s.r + kWarpsH - 1) / kWarpsH) * ((s.T + TT - 1) / TT);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  e = launch_pdl(kern, dim3((unsigned)blocks), dim3(kThreadsH), smem, st, (const char *)x,
                 (const char *)A, h, s.T, s.d, s.r, (const char *)pf, (int64_t)pf_bytes);
  count_launches(1);
  return e;
}

template <class E, int TT, bool W, bool K, bool SB>
cudaError_t logits_tt(const FwdShape &s, const float *h, const void *B, float *logits,
                      uint64_t *mask, int *sel_idx, float *sel_sig, unsigned *err,
                      cudaStream_t st) {
  const size_t block = SB ? (size_t)s.bank * s.r * E::kBytes : 0;
  const size_t smem = block + (size_t)TT * (s.r + 128) * sizeof(float) + 16;
  auto kern = k_logits_topk<E, TT, W, K, SB>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)s.n_banks * ((s.T + TT - 1) / TT);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  e = launch_pdl(kern, dim3((unsigned)blocks), dim3(kThreads), smem, st, h, (const char *)B,
                 logits, mask, sel_idx, sel_sig, s.T, s.d_i, s.r, s.bank, s.k, err);
  count_launches(1);
  return e;
}

template <class E, bool W, bool K>
cudaError_t logits_dispatch(const FwdShape &s, int tt, const float *h, const void *B,
                            float *logits, uint64_t *mask, int *sel_idx, float *sel_sig,
                            unsigned *err, cudaStream_t st) {
  const bool sb = (size_t)s.bank * s.r * E::kBytes <= kMaxBBlock;
#define SFN_LT(TTV)                                                                      \
  return sb ? logits_tt<E, TTV, W, K, true>(s, h, B, logits, mask, sel_idx, sel_sig, err, st) \
            : logits_tt<E, TTV, W, K, false>(s, h, B, logits, mask, sel_idx, sel_sig, err, st)
  switch (tt) {
    case 1: SFN_LT(1);
    case 2: SFN_LT(2);
    case 4: SFN_LT(4);
    default: SFN_LT(8);
  }
#undef SFN_LT
}

}  // namespace

cudaError_t launch_pred_h(const FwdShape &s, int tt, const void *x, const void *A, void *h,
                          bool split_out, cudaStream_t st, const void *prefetch,
                          size_t prefetch_bytes) {
#define SFN_PH(ELT, TTV)                                                                     \
  return split_out ? pred_h_tt<ELT, TTV, true>(s, x, A, h, prefetch, prefetch_bytes, st) \
                   : pred_h_tt<ELT, TTV, false>(s, x, A, h, prefetch, prefetch_bytes, st)
  if (s.bf16) {
    switch (tt) {
      case 1: SFN_PH(EltBF16, 1);
      case 2: SFN_PH(EltBF16, 2);
      case 4: SFN_PH(EltBF16, 4);
      default: SFN_PH(EltBF16, 8);
    }
  }
  switch (tt) {
    case 1: SFN_PH(EltF32, 1);
    case 2: SFN_PH(EltF32, 2);
    case 4: SFN_PH(EltF32, 4);
    default: SFN_PH(EltF32, 8);
  }
#undef SFN_PH
}

cudaError_t launch_logits_topk(const FwdShape &s, int tt, const float *h, const void *B,
                               float *logits, uint64_t *mask, int *sel_idx, float *sel_sig,
                               unsigned *err, cudaStream_t st) {
  const bool topk = sel_idx != nullptr;
  const bool write = logits != nullptr;
  if (s.bf16) {
    if (topk && write)
      return logits_dispatch<EltBF16, true, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
    if (topk)
      return logits_dispatch<EltBF16, false, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
    return logits_dispatch<EltBF16, true, false>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
  }
  if (topk && write)
    return logits_dispatch<EltF32, true, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
  if (topk)
    return logits_dispatch<EltF32, false, true>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
  return logits_dispatch<EltF32, true, false>(s, tt, h, B, logits, mask, sel_idx, sel_sig, err, st);
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
