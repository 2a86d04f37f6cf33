// gather_ffn.cu -- sparse gate/up/down over the kept channels only, on CUDA
// cores (the few-token path).
//
// "Inactive channels are exactly zero" and the gate, up and down projections
// skip them: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
// Training Recipe for Dense-to-Sparse LLMs", gist.science summary,
// "1. Architectuur" (Executie / Forward Pass) and "3. Hardware Implicaties".
//
//   k_gateup_ring  the kept (token, slot) pairs are split evenly over the
//                  CTAs.  In each CTA one producer thread streams the kept
//                  W_gate and W_up rows into an 8-stage shared-memory ring
//                  with 1-D bulk (TMA) copies; 8 consumer warps each own one
//                  stage and compute g = Wg[j].x, u = Wu[j].x and
//                  a = sigma(p_j) g u.  The producer also prefetches the
//                  kept W_down row into L2 for k_down_slices.
//   k_down_slices  y[t][cols] = sum over the kept slots of a * Wd[j][cols],
//                  one CTA per (token, 32-column slice), slots summed in a
//                  fixed order (deterministic), rows read from L2.
// Only the kept rows of Wg, Wu and Wd are ever read.
#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kMaxStages = 8;          // ring stages = consumer warps (one each)
constexpr size_t kRingBudget = 200 * 1024;  // shared memory for the ring
constexpr int kDownThreads = 256;
constexpr int kSliceCols = 32;

// blockDim.x = (n_stages + 1) * 32: warps 0..n_stages-1 consume, the last
// warp produces.
template <class E>
__global__ void __launch_bounds__((kMaxStages + 1) * 32) k_gateup_ring(
    const char *__restrict__ x, const int *__restrict__ sel_idx,
    const float *__restrict__ sel_sig, const char *__restrict__ Wg,
    const char *__restrict__ Wu, const char *__restrict__ Wd, float *__restrict__ a_out,
    int64_t n_slots, int d_s, int d, int n_stages, unsigned *err) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t row_bytes = (uint32_t)d * E::kBytes;
  const int kConsumerWarps = n_stages;
  unsigned char *ring = smem;  // [n_stages][2][row_bytes]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)n_stages * 2 * row_bytes);
  uint64_t *empty = full + kMaxStages;

  // this CTA's contiguous range of flattened slots f = t * d_s + s
  const int64_t per = n_slots / gridDim.x, rem = n_slots % gridDim.x;
  const int64_t f0 = blockIdx.x * per + (blockIdx.x < rem ? blockIdx.x : rem);
  const int64_t cnt = per + (blockIdx.x < rem ? 1 : 0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kConsumerWarps; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // sel_idx, sel_sig and x come from earlier work on the stream

  if (warp == kConsumerWarps) {
    // producer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t n = 0; n < cnt; ++n) {
        const int st = (int)(n % kConsumerWarps);
        const uint32_t use = (uint32_t)(n / kConsumerWarps);
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1u, err)) break;
        const int64_t j = sel_idx[f0 + n];
        unsigned char *dst = ring + (size_t)st * 2 * row_bytes;
        mbar_arrive_expect_tx(&full[st], 2 * row_bytes);
        bulk_g2s(dst, Wg + j * row_bytes, row_bytes, &full[st]);
        bulk_g2s(dst + row_bytes, Wu + j * row_bytes, row_bytes, &full[st]);
        prefetch_l2(Wd + j * row_bytes, row_bytes);
        issued = n + 1;
      }
      // Do not leave while a copy may still be landing in shared memory:
      // wait (bounded) for the last issued use of every stage.
      for (int st = 0; st < kConsumerWarps; ++st) {
        if (issued <= st) break;
        const int64_t last = st + ((issued - 1 - st) / kConsumerWarps) * kConsumerWarps;
        mbar_wait(&full[st], (uint32_t)(last / kConsumerWarps) & 1u, err);
      }
    }
    return;
  }

  // consumer warp `warp` owns stage `warp`: slots n = warp, warp + 8, ...
  const int nchunk = d / E::kVec;
  const unsigned char *gs = ring + (size_t)warp * 2 * row_bytes;
  const unsigned char *us = gs + row_bytes;
  for (int64_t n = warp; n < cnt; n += kConsumerWarps) {
    if (!mbar_wait(&full[warp], (uint32_t)(n / kConsumerWarps) & 1u, err)) break;
    const int64_t f = f0 + n;
    const int64_t t = f / d_s;
    const char *xr = x + t * d * E::kBytes;
    float g = 0.f, u = 0.f;
#pragma unroll 4
    for (int q = lane; q < nchunk; q += 32) {
      float wg[E::kVec], wu[E::kVec], xv[E::kVec];
      E::unpack(*reinterpret_cast<const uint4 *>(gs + (size_t)q * 16), wg);
      E::unpack(*reinterpret_cast<const uint4 *>(us + (size_t)q * 16), wu);
      E::unpack(ld_nc16(xr + (size_t)q * 16), xv);
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) {
        g = fmaf(wg[e], xv[e], g);
        u = fmaf(wu[e], xv[e], u);
      }
    }
    g = warp_sum(g);
    u = warp_sum(u);
    __syncwarp();
    if (lane == 0) {
      a_out[f] = sel_sig[f] * g * u;
      mbar_arrive(&empty[warp]);
    }
  }
}

// y[t][c0 .. c0+31] = sum_s a[t][s] * Wd[sel_idx[t][s]][c0 .. c0+31].
// blockIdx.x = t * n_slices + slice.  A lane reads one 16-byte chunk of one
// slot's row slice; lanes sharing a chunk index split the slots, and the
// partial sums are combined in a fixed order (shuffles, then warps in order).
template <class E>
__global__ void __launch_bounds__(kDownThreads) k_down_slices(
    const int *__restrict__ sel_idx, const float *__restrict__ a, const char *__restrict__ Wd,
    void *__restrict__ y, int d, int d_s, int n_slices) {
  constexpr int kCpr = kSliceCols / E::kVec;  // 16-byte chunks per slice row
  constexpr int kRpw = 32 / kCpr;             // slot rows per warp instruction
  __shared__ float red[kDownThreads / 32][kSliceCols];
  const int64_t t = blockIdx.x / n_slices;
  const int c0 = (blockIdx.x % n_slices) * kSliceCols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / kCpr, cc = lane % kCpr;
  const int col = c0 + cc * E::kVec;
  const bool col_ok = col < d;  // d is a multiple of kVec
  pdl_launch_dependents();
  pdl_wait();

  const int *idx = sel_idx + t * d_s;
  const float *av = a + t * d_s;
  float acc[E::kVec];
#pragma unroll
  for (int e = 0; e < E::kVec; ++e) acc[e] = 0.f;
  constexpr int kStride = (kDownThreads / 32) * kRpw;  // slots per CTA sweep
  int s = warp * kRpw + sub;
  // 8 independent row loads in flight per lane per batch
  for (; s + 7 * kStride < d_s; s += 8 * kStride) {
    uint4 v[8];
    float w8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = idx[s + u * kStride];
      w8[u] = av[s + u * kStride];
      v[u] = col_ok ? ld_nc16(Wd + (j * d + col) * E::kBytes) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float w[E::kVec];
      E::unpack(v[u], w);
#pragma unroll
      for (int e = 0; e < E::kVec; ++e) acc[e] = fmaf(w8[u], w[e], acc[e]);
    }
  }
  for (; s < d_s; s += kStride) {
    const int64_t j = idx[s];
    const float wa = av[s];
    float w[E::kVec];
    E::unpack(col_ok ? ld_nc16(Wd + (j * d + col) * E::kBytes) : make_uint4(0, 0, 0, 0), w);
#pragma unroll
    for (int e = 0; e < E::kVec; ++e) acc[e] = fmaf(wa, w[e], acc[e]);
  }
  // combine lanes with the same chunk index (fixed butterfly order)
#pragma unroll
  for (int o = kCpr; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < E::kVec; ++e) acc[e] += __shfl_xor_sync(kFull, acc[e], o);
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < E::kVec; ++e) red[warp][cc * E::kVec + e] = acc[e];
  }
  __syncthreads();
  if (threadIdx.x < kSliceCols) {
    const int c = c0 + threadIdx.x;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDownThreads / 32; ++w) v += red[w][threadIdx.x];
    if (c < d) {
      if (E::kBytes == 2)
        reinterpret_cast<uint16_t *>(y)[t * d + c] = f32_to_bf16_bits(v);
      else
        reinterpret_cast<float *>(y)[t * d + c] = v;
    }
  }
}

}  // namespace
size_t gateup_smem_bytes(const FwdShape &s);
namespace {

int gateup_stages(const FwdShape &s) {
  const size_t stage = (size_t)2 * s.d * (s.bf16 ? 2 : 4);
  int n = (int)(kRingBudget / stage);
  return n < 1 ? 1 : (n > kMaxStages ? kMaxStages : n);
}

template <class E>
cudaError_t gateup_e(const FwdShape &s, int ctas, const void *x, const int *sel_idx,
                     const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                     float *a_out, unsigned *err, cudaStream_t st) {
  const int n_stages = gateup_stages(s);
  const size_t smem = gateup_smem_bytes(s);
  auto kern = k_gateup_ring<E>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(ctas), dim3((n_stages + 1) * 32), smem, st, (const char *)x,
                 sel_idx, sel_sig, (const char *)Wg, (const char *)Wu, (const char *)Wd, a_out,
                 (int64_t)s.T * s.d_s, s.d_s, s.d, n_stages, err);
  count_launches(1);
  return e;
}

template <class E>
cudaError_t down_e(const FwdShape &s, const int *sel_idx, const float *a, const void *Wd,
                   void *y, cudaStream_t st) {
  const int n_slices = (s.d + kSliceCols - 1) / kSliceCols;
  const int64_t blocks = (int64_t)n_slices * s.T;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e = launch_pdl(k_down_slices<E>, dim3((unsigned)blocks), dim3(kDownThreads), 0,
                             st, sel_idx, a, (const char *)Wd, y, s.d, s.d_s, n_slices);
  count_launches(1);
  return e;
}

}  // namespace

size_t gateup_smem_bytes(const FwdShape &s) {
  return (size_t)gateup_stages(s) * 2 * s.d * (s.bf16 ? 2 : 4) + 2 * kMaxStages * sizeof(uint64_t);
}

cudaError_t launch_gateup(const FwdShape &s, int ctas, const void *x, const int *sel_idx,
                          const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                          float *a_out, unsigned *err, cudaStream_t st) {
  if (s.bf16) return gateup_e<EltBF16>(s, ctas, x, sel_idx, sel_sig, Wg, Wu, Wd, a_out, err, st);
  return gateup_e<EltF32>(s, ctas, x, sel_idx, sel_sig, Wg, Wu, Wd, a_out, err, st);
}

cudaError_t launch_down(const FwdShape &s, const int *sel_idx, const float *a, const void *Wd,
                        void *y, cudaStream_t st) {
  if (s.bf16) return down_e<EltBF16>(s, sel_idx, a, Wd, y, st);
  return down_e<EltF32>(s, sel_idx, a, Wd, y, st);
}

}  // namespace sfn
