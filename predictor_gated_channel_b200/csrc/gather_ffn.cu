// gather_ffn.cu -- sparse gate/up/down over the kept channels only, on CUDA
// cores (the few-token path).
//
// "Inactive channels are exactly zero" and the gate, up and down projections
// skip them: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
// Training Recipe for Dense-to-Sparse LLMs", gist.science summary,
// "1. Architectuur" (Executie / Forward Pass) and "3. Hardware Implicaties".
//
//   k_gather_ffn  one CTA per (token, chunk of kept-channel slots):
//                 phase A, a warp per slot: g = Wg[j].x, u = Wu[j].x,
//                 a = sigma(p_j) g u; phase B, every thread owns 16-byte
//                 column chunks of the output and accumulates a_j Wd[j, :]
//                 over the chunk's slots in slot order -> fp32 partial row.
//   k_reduce      y[t] = sum over chunks of the partial rows, in chunk order,
//                 rounded to the output type.
// Only the kept rows of Wg, Wu and Wd are ever read.
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <class E>
__global__ void __launch_bounds__(kThreads) k_gather_ffn(
    const char *__restrict__ x, const int *__restrict__ sel_idx,
    const float *__restrict__ sel_sig, const char *__restrict__ Wg,
    const char *__restrict__ Wu, const char *__restrict__ Wd, float *__restrict__ partial,
    int d, int d_s, int n_chunks, int chunk) {
  extern __shared__ float4 smem_f4[];
  float *xs = reinterpret_cast<float *>(smem_f4);  // [d]
  float *as = xs + d;                              // [chunk]
  int *js = reinterpret_cast<int *>(as + chunk);   // [chunk]

  const int64_t t = blockIdx.x / n_chunks;
  const int c = blockIdx.x % n_chunks;
  const int s0 = c * chunk;
  const int ns = min(chunk, d_s - s0);
  const int nchunk = d / E::kVec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < nchunk; i += blockDim.x) {
    float f[E::kVec];
    E::unpack(ld_nc16(x + (t * d + (int64_t)i * E::kVec) * E::kBytes), f);
    float4 *dst = reinterpret_cast<float4 *>(xs + i * E::kVec);
#pragma unroll
    for (int e = 0; e < E::kVec / 4; ++e)
      dst[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
  }
  for (int i = threadIdx.x; i < ns; i += blockDim.x) js[i] = sel_idx[t * d_s + s0 + i];
  __syncthreads();

  // Phase A: gate and up dot products of the kept channels.
  for (int i = warp; i < ns; i += kWarps) {
    const int64_t j = js[i];
    const char *grow = Wg + j * d * E::kBytes;
    const char *urow = Wu + j * d * E::kBytes;
    float g = 0.f, u = 0.f;
#pragma unroll 4
    for (int q = lane; q < nchunk; q += 32) {
      float wg[E::kVec], wu[E::kVec];
      E::unpack(ld_stream16(grow + (int64_t)q * 16), wg);
      E::unpack(ld_stream16(urow + (int64_t)q * 16), wu);
      const float *xr = xs + q * E::kVec;
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) {
        g = fmaf(wg[e], xr[e], g);
        u = fmaf(wu[e], xr[e], u);
      }
    }
    g = warp_sum(g);
    u = warp_sum(u);
    if (lane == 0) as[i] = sel_sig[t * d_s + s0 + i] * g * u;
  }
  __syncthreads();

  // Phase B: partial[t][c][:] = sum_i as[i] * Wd[js[i], :], slots in order.
  float *out = partial + (t * n_chunks + c) * (int64_t)d;
  for (int q = threadIdx.x; q < nchunk; q += blockDim.x) {
    float acc[E::kVec];
#pragma unroll
    for (int e = 0; e < E::kVec; ++e) acc[e] = 0.f;
#pragma unroll 8
    for (int i = 0; i < ns; ++i) {
      float w[E::kVec];
      E::unpack(ld_stream16(Wd + ((int64_t)js[i] * d + (int64_t)q * E::kVec) * E::kBytes), w);
      const float a = as[i];
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) acc[e] = fmaf(a, w[e], acc[e]);
    }
    float4 *dst = reinterpret_cast<float4 *>(out + q * E::kVec);
#pragma unroll
    for (int e = 0; e < E::kVec / 4; ++e)
      dst[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
  }
}

// y[t][n..n+3] = sum_c partial[t][c][n..n+3].  1-D grid:
// blockIdx.x = t * col_blocks + col_block, col_blocks = ceil(d / 4 / 256).
template <bool kBF16>
__global__ void __launch_bounds__(kThreads) k_reduce(const float *__restrict__ partial,
                                                     void *__restrict__ y, int d,
                                                     int n_chunks) {
  const int col_blocks = (d / 4 + kThreads - 1) / kThreads;
  const int64_t t = blockIdx.x / col_blocks;
  const int n = ((blockIdx.x % col_blocks) * kThreads + threadIdx.x) * 4;
  if (n >= d) return;
  const float *p = partial + t * n_chunks * (int64_t)d + n;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < n_chunks; ++c) {
    const float4 v = *reinterpret_cast<const float4 *>(p + (int64_t)c * d);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  if (kBF16) {
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(y) + t * d + n) = o;
  } else {
    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + t * d + n) = acc;
  }
}

template <class E>
cudaError_t gather_e(const FwdShape &s, const GatherPlan &p, const void *x, const int *sel_idx,
                     const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                     float *partial, cudaStream_t st) {
  const size_t smem = (size_t)s.d * sizeof(float) + (size_t)p.chunk * 8;
  auto kern = k_gather_ffn<E>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.n_chunks * s.T;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<(unsigned)blocks, kThreads, smem, st>>>((const char *)x, sel_idx, sel_sig, (const char *)Wg,
                                     (const char *)Wu, (const char *)Wd, partial, s.d, s.d_s,
                                     p.n_chunks, p.chunk);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather_ffn(const FwdShape &s, const GatherPlan &p, const void *x,
                              const int *sel_idx, const float *sel_sig, const void *Wg,
                              const void *Wu, const void *Wd, float *partial,
                              cudaStream_t st) {
  if (s.bf16) return gather_e<EltBF16>(s, p, x, sel_idx, sel_sig, Wg, Wu, Wd, partial, st);
  return gather_e<EltF32>(s, p, x, sel_idx, sel_sig, Wg, Wu, Wd, partial, st);
}

cudaError_t launch_reduce(const FwdShape &s, const GatherPlan &p, const float *partial,
                          void *y, cudaStream_t st) {
  const int64_t blocks = (int64_t)((s.d / 4 + kThreads - 1) / kThreads) * s.T;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (s.bf16)
    k_reduce<true><<<(unsigned)blocks, kThreads, 0, st>>>(partial, y, s.d, p.n_chunks);
  else
    k_reduce<false><<<(unsigned)blocks, kThreads, 0, st>>>(partial, y, s.d, p.n_chunks);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace sfn
