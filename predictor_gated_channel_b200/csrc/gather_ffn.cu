// gather_ffn.cu -- sparse gate/up/down over the kept channels only, on CUDA
// cores (the few-token path).
//
// Channels outside the mask are exactly zero in the forward pass, so the gate,
// up and down projections may skip them: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
// Training Recipe for Dense-to-Sparse LLMs", gist.science summary,
// "1. Architectuur" (Executie / Forward Pass) and "3. Hardware Implicaties".
//
//   k_ffn_ring         one CTA per (token, contiguous range of its kept slots).
//                      A producer warp streams, for every slot, the kept
//                      W_gate, W_up and W_down rows into shared-memory rings
//                      with 1-D bulk (TMA) copies, one issuing lane per ring
//                      stage.  S gate/up warps (one per
//                      ring stage) compute g = Wg[j].x, u = Wu[j].x and
//                      a = sigma(p_j) g u and hand a to 8 down warps; each
//                      down warp owns one eighth of the output columns in
//                      registers and accumulates a * Wd[j, cols] over the
//                      slots in order.  The CTA writes one fp32 partial row.
//   k_reduce_partials  y[t] = sum of the token's partial rows in a fixed
//                      order, rounded to the output type.  Also the tensor
//                      path's split-K sums (fp32 partials of h and of y).
//   k_reduce_few       the same for at most 16 partials: one thread per four
//                      columns, no shared memory.
// Only the kept rows of Wg, Wu and Wd are read, each once per token; all sums
// run in a fixed order, so results are bit-reproducible.
#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kMaxStages = 8;   // ring stages = gate/up warps (one each)
constexpr int kDownWarps = 8;   // output column eighths
constexpr int kMaxChunks = 4;   // 16-byte column chunks per down lane
// 7 stages of 24 KB rows (d = 4096, bf16): leaves room on the SM for the
// next call's h kernel, which prefetches the predictor weights meanwhile
constexpr size_t kRingBudget = 168 * 1024;
constexpr int kMaxSlotsPerCta = 1024;
constexpr uint32_t kMaxXBytes = 16384;  // one token row of x staged in smem
constexpr int kReduceThreads = 256;

struct RingLayout {
  uint32_t row_bytes;
  int stages;
  size_t off_gu, off_d, off_a, off_idx, off_sig, off_x, off_bar, total;
};

__host__ __device__ inline RingLayout ring_layout(int d, int elt_bytes) {
  RingLayout L;
  L.row_bytes = (uint32_t)d * elt_bytes;
  int s = (int)(kRingBudget / (3ull * L.row_bytes));
  L.stages = s < 1 ? 1 : (s > kMaxStages ? kMaxStages : s);
  L.off_gu = 0;
  L.off_d = L.off_gu + (size_t)L.stages * 2 * L.row_bytes;
  L.off_a = L.off_d + (size_t)L.stages * L.row_bytes;
  L.off_idx = L.off_a + (size_t)kMaxSlotsPerCta * sizeof(float);
  L.off_sig = L.off_idx + (size_t)kMaxSlotsPerCta * sizeof(int);
  L.off_x = L.off_sig + (size_t)kMaxSlotsPerCta * sizeof(float);
  L.off_bar = L.off_x + kMaxXBytes;
  L.total = L.off_bar + 5 * kMaxStages * sizeof(uint64_t);
  return L;
}

// blockDim.x = (stages + kDownWarps + 1) * 32: warps [0, S) gate/up,
// [S, S + 8) down, the last warp produces.  blockIdx.x = t * cpt + c.
template <class E>
__global__ void __launch_bounds__((kMaxStages + kDownWarps + 1) * 32, 1)
    k_ffn_ring(const char *__restrict__ x, const int *__restrict__ sel_idx,
               const float *__restrict__ sel_sig, const char *__restrict__ Wg,
               const char *__restrict__ Wu, const char *__restrict__ Wd,
               float *__restrict__ partial, int d_s, int d, int cpt, unsigned *err) {
  extern __shared__ __align__(128) unsigned char smem[];
  const RingLayout L = ring_layout(d, E::kBytes);
  const int S = L.stages;
  unsigned char *gu_ring = smem + L.off_gu;  // [S][2][row]
  unsigned char *d_ring = smem + L.off_d;    // [S][row]
  float *a_s = reinterpret_cast<float *>(smem + L.off_a);
  int *idx_s = reinterpret_cast<int *>(smem + L.off_idx);
  float *sig_s = reinterpret_cast<float *>(smem + L.off_sig);
  unsigned char *x_s = smem + L.off_x;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.off_bar);
  uint64_t *gu_full = bar, *gu_empty = bar + kMaxStages, *d_full = bar + 2 * kMaxStages;
  uint64_t *d_empty = bar + 3 * kMaxStages, *a_ready = bar + 4 * kMaxStages;

  const int64_t t = blockIdx.x / cpt;
  const int c = blockIdx.x % cpt;
  const int s0 = (int)(((int64_t)d_s * c) / cpt);
  const int cnt = (int)(((int64_t)d_s * (c + 1)) / cpt) - s0;
  const int64_t f0 = t * d_s + s0;  // flattened index of the first slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&gu_full[i], 1);
      mbar_init(&gu_empty[i], 1);
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kDownWarps);
      mbar_init(&a_ready[i], 1);
    }
    fence_barrier_init();
  }
  pdl_wait();  // sel_idx and sel_sig come from the previous kernel
  pdl_launch_dependents();
  // stage this CTA's kept channel ids, their sigma(p) and the token's x;
  // each thread issues its loads before its stores (one round trip)
  const uint32_t row = L.row_bytes;
  const int nx = (int)(row / 16);
  for (int i = threadIdx.x; i < cnt || i < nx; i += blockDim.x) {
    int j = 0;
    float sg = 0.f;
    uint4 xv = make_uint4(0, 0, 0, 0);
    if (i < cnt) {
      j = sel_idx[f0 + i];
      sg = sel_sig[f0 + i];
    }
    if (i < nx) xv = ld_nc16(x + t * row + (size_t)i * 16);
    if (i < cnt) {
      idx_s[i] = j;
      sig_s[i] = sg;
    }
    if (i < nx) *reinterpret_cast<uint4 *>(x_s + (size_t)i * 16) = xv;
  }
  __syncthreads();

  if (warp == S + kDownWarps) {
    // ----------------------------------------------------------- producer
    // Lane st owns ring stage st and issues the copies of slots st, st + S,
    // ...: several independent issuers keep more row fetches in flight than
    // one thread issuing every copy in turn.
    const int st = lane;
    // kept rows are read once: evict them from L2 first, ahead of the next
    // call's predictor weights that its first kernel prefetches meanwhile
    const uint64_t once = make_evict_first_policy();
    if (st < S) {
      int issued = 0;
      for (int n = st; n < cnt; n += S) {
        const uint32_t use = (uint32_t)(n / S);
        if (use > 0 && (!mbar_wait(&gu_empty[st], (use - 1) & 1u, err) ||
                        !mbar_wait(&d_empty[st], (use - 1) & 1u, err)))
          break;
        const int64_t j = idx_s[n];
        unsigned char *gdst = gu_ring + (size_t)st * 2 * row;
        mbar_arrive_expect_tx(&gu_full[st], 2 * row);
        bulk_g2s_hint(gdst, Wg + j * row, row, &gu_full[st], once);
        bulk_g2s_hint(gdst + row, Wu + j * row, row, &gu_full[st], once);
        mbar_arrive_expect_tx(&d_full[st], row);
        bulk_g2s_hint(d_ring + (size_t)st * row, Wd + j * row, row, &d_full[st], once);
        issued = use + 1;
      }
      // never leave while a copy may still be landing in shared memory
      if (issued > 0) {
        mbar_wait(&gu_full[st], (uint32_t)(issued - 1) & 1u, err);
        mbar_wait(&d_full[st], (uint32_t)(issued - 1) & 1u, err);
      }
    }
    return;
  }

  if (warp < S) {
    // ----------------------------------------------------------- gate / up
    const int nchunk = d / E::kVec;
    const unsigned char *gs = gu_ring + (size_t)warp * 2 * row;
    const unsigned char *us = gs + row;
    for (int n = warp; n < cnt; n += S) {
      if (!mbar_wait(&gu_full[warp], (uint32_t)(n / S) & 1u, err)) break;
      float g = 0.f, u = 0.f;
#pragma unroll 4
      for (int q = lane; q < nchunk; q += 32) {
        float wg[E::kVec], wu[E::kVec], xv[E::kVec];
        E::unpack(*reinterpret_cast<const uint4 *>(gs + (size_t)q * 16), wg);
        E::unpack(*reinterpret_cast<const uint4 *>(us + (size_t)q * 16), wu);
        E::unpack(*reinterpret_cast<const uint4 *>(x_s + (size_t)q * 16), xv);
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
        a_s[n] = sig_s[n] * g * u;
        mbar_arrive(&gu_empty[warp]);
        mbar_arrive(&a_ready[warp]);
      }
    }
    return;
  }

  // ------------------------------------------------------------- down
  const int dw = warp - S;
  const int nq = d / E::kVec / kDownWarps;  // 16-byte chunks per down warp
  float acc[kMaxChunks][E::kVec];
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i)
#pragma unroll
    for (int e = 0; e < E::kVec; ++e) acc[i][e] = 0.f;
  for (int n = 0; n < cnt; ++n) {
    const int st = n % S;
    const uint32_t par = (uint32_t)(n / S) & 1u;
    if (!mbar_wait(&d_full[st], par, err) || !mbar_wait(&a_ready[st], par, err)) break;
    const float a = a_s[n];
    const unsigned char *wr = d_ring + (size_t)st * row + (size_t)dw * nq * 16;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
      const int q = lane + 32 * i;
      if (q < nq) {
        float w[E::kVec];
        E::unpack(*reinterpret_cast<const uint4 *>(wr + (size_t)q * 16), w);
#pragma unroll
        for (int e = 0; e < E::kVec; ++e) acc[i][e] = fmaf(a, w[e], acc[i][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&d_empty[st]);
  }
  float *out = partial + ((t * cpt) + c) * (int64_t)d + (int64_t)dw * nq * E::kVec;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int q = lane + 32 * i;
    if (q < nq) {
      float4 *dst = reinterpret_cast<float4 *>(out + (size_t)q * E::kVec);
#pragma unroll
      for (int e = 0; e < E::kVec / 4; ++e)
        dst[e] = make_float4(acc[i][4 * e], acc[i][4 * e + 1], acc[i][4 * e + 2], acc[i][4 * e + 3]);
    }
  }
}

// out[t][c0 .. c0+C) = sum_{c < cpt} partial[t][c][c0 .. c0+C), summed in a
// fixed order.  blockIdx.x = t * ceil(n / C) + slice.  Thread = (group g,
// quad q), q fastest: group g sums partials c = g, g + G, ... (its loads
// issued as one batch of kBatch); the four groups of a warp that share q are
// combined by two shuffles, then the warps' sums in warp order.  kOut: 0 =
// float32 out, 1 = bf16 out, 2 = bf16 hi/lo halves of h ([T][2n]: hi at
// column j, lo = bf16(sum - hi) at n + j).
template <int C, int kOut>
__global__ void __launch_bounds__(kReduceThreads) k_reduce_partials(
    const float *__restrict__ partial, void *__restrict__ out, int n, int cpt) {
  constexpr int Q = C / 4;                // float4 quads per slice
  constexpr int G = kReduceThreads / Q;   // partial groups
  constexpr int kWarps = kReduceThreads / 32;
  constexpr int kBatch = 8;               // loads per thread in flight
  static_assert(Q == 8 || Q == 32, "a warp holds 4 groups of 8 quads or 1 group of 32");
  __shared__ float4 red[kWarps][Q];
  const int slices = (n + C - 1) / C;
  const int64_t t = blockIdx.x / slices;
  const int c0 = (blockIdx.x % slices) * C;
  const int g = threadIdx.x / Q, q = threadIdx.x % Q;
  const int col = c0 + q * 4;
  // The stream's next kernel is released once the partials are complete, not
  // earlier.  As the last kernel of a CUDA-core forward call, this puts the
  // next call's prologue (its L2 prefetch of the predictor's B) in DRAM's
  // idle time here rather than in the bandwidth-bound gate/up/down kernel.
  pdl_wait();
  pdl_launch_dependents();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col < n) {
    const float *p = partial + t * cpt * (int64_t)n + col;
    for (int cb = g; cb < cpt; cb += kBatch * G) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        v[u] = (cb + u * G < cpt) ? *reinterpret_cast<const float4 *>(p + (int64_t)(cb + u * G) * n)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        acc.x += v[u].x;
        acc.y += v[u].y;
        acc.z += v[u].z;
        acc.w += v[u].w;
      }
    }
  }
  // lanes q, q + 8, q + 16, q + 24 of a warp hold groups of the same quad
  if (Q == 8) {
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < Q) red[warp][lane] = acc;
  __syncthreads();
  if (threadIdx.x < Q) {
    float4 v = red[0][threadIdx.x];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      const float4 r4 = red[w][threadIdx.x];
      v.x += r4.x;
      v.y += r4.y;
      v.z += r4.z;
      v.w += r4.w;
    }
    const int cc = c0 + threadIdx.x * 4;
    if (cc < n) {
      if (kOut == 0) {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + t * n + cc) = v;
      } else if (kOut == 1) {
        uint2 o;
        o.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
        o.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
        *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(out) + t * n + cc) = o;
      } else {
        const float f[4] = {v.x, v.y, v.z, v.w};
        uint16_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = f32_to_bf16_bits(f[e]);
          lo[e] = f32_to_bf16_bits(f[e] - __uint_as_float((uint32_t)hi[e] << 16));
        }
        uint16_t *h2 = reinterpret_cast<uint16_t *>(out) + t * 2 * n;
        *reinterpret_cast<uint2 *>(h2 + cc) =
            make_uint2(hi[0] | ((uint32_t)hi[1] << 16), hi[2] | ((uint32_t)hi[3] << 16));
        *reinterpret_cast<uint2 *>(h2 + n + cc) =
            make_uint2(lo[0] | ((uint32_t)lo[1] << 16), lo[2] | ((uint32_t)lo[3] << 16));
      }
    }
  }
}

// Four consecutive outputs v at out[i .. i + 4): kOut 0 float32, 1 bf16.
template <int kOut>
__device__ __forceinline__ void store_quad(void *out, int64_t i, float4 v) {
  if (kOut == 0) {
    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + i) = v;
  } else {
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(out) + i) = o;
  }
}

// Few partials (cpt <= kSmallCpt): one thread per four columns adds the cpt
// partial rows in order 0, 1, ..., with its loads in flight together.  No
// shared memory, so its CTAs fit beside a large-shared-memory kernel still
// running on the SM and start early (programmatic dependent launch).
constexpr int kSmallCpt = 16;
template <int kOut>
__global__ void __launch_bounds__(kReduceThreads) k_reduce_few(
    const float *__restrict__ partial, void *__restrict__ out, int n, int cpt) {
  const int per_t = (n / 4 + kReduceThreads - 1) / kReduceThreads;
  const int64_t t = blockIdx.x / per_t;
  const int col = ((blockIdx.x % per_t) * kReduceThreads + threadIdx.x) * 4;
  pdl_wait();
  pdl_launch_dependents();
  if (col >= n) return;
  const float *p = partial + t * cpt * (int64_t)n + col;
  float4 v[kSmallCpt];
#pragma unroll
  for (int c = 0; c < kSmallCpt; ++c)
    v[c] = (c < cpt) ? *reinterpret_cast<const float4 *>(p + (int64_t)c * n)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 acc = v[0];
#pragma unroll
  for (int c = 1; c < kSmallCpt; ++c) {
    if (c < cpt) {
      acc.x += v[c].x;
      acc.y += v[c].y;
      acc.z += v[c].z;
      acc.w += v[c].w;
    }
  }
  if (kOut == 0 || kOut == 1) {
    store_quad<kOut == 0 ? 0 : 1>(out, t * n + col, acc);
  } else {
    const float f[4] = {acc.x, acc.y, acc.z, acc.w};
    uint16_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      hi[e] = f32_to_bf16_bits(f[e]);
      lo[e] = f32_to_bf16_bits(f[e] - __uint_as_float((uint32_t)hi[e] << 16));
    }
    uint16_t *h2 = reinterpret_cast<uint16_t *>(out) + t * 2 * n;
    *reinterpret_cast<uint2 *>(h2 + col) =
        make_uint2(hi[0] | ((uint32_t)hi[1] << 16), hi[2] | ((uint32_t)hi[3] << 16));
    *reinterpret_cast<uint2 *>(h2 + n + col) =
        make_uint2(lo[0] | ((uint32_t)lo[1] << 16), lo[2] | ((uint32_t)lo[3] << 16));
  }
}

template <class E>
cudaError_t ffn_e(const FwdShape &s, int cpt, const void *x, const int *sel_idx,
                  const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                  float *partial, unsigned *err, cudaStream_t st) {
  const RingLayout L = ring_layout(s.d, E::kBytes);
  auto kern = k_ffn_ring<E>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), L.total);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)cpt * s.T;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  e = launch_pdl(kern, dim3((unsigned)blocks), dim3((L.stages + kDownWarps + 1) * 32), L.total,
                 st, (const char *)x, sel_idx, sel_sig, (const char *)Wg, (const char *)Wu,
                 (const char *)Wd, partial, s.d_s, s.d, cpt, err);
  count_launches(1);
  return e;
}

}  // namespace

bool ffn_shape_ok(const FwdShape &s) {
  const int elt = s.bf16 ? 2 : 4;
  const int vec = 16 / elt;
  return s.d % (vec * kDownWarps) == 0 && s.d / vec / kDownWarps <= 32 * kMaxChunks &&
         (uint32_t)s.d * elt <= kMaxXBytes;
}

int ffn_ctas_per_token(const FwdShape &s, int num_sms) {
  int64_t cpt = num_sms / s.T;
  if (cpt < 1) cpt = 1;
  const int64_t min_cpt = (s.d_s + kMaxSlotsPerCta - 1) / kMaxSlotsPerCta;
  if (cpt < min_cpt) cpt = min_cpt;
  if (cpt > s.d_s) cpt = s.d_s;
  return (int)cpt;
}

cudaError_t launch_ffn(const FwdShape &s, int cpt, const void *x, const int *sel_idx,
                       const float *sel_sig, const void *Wg, const void *Wu, const void *Wd,
                       float *partial, unsigned *err, cudaStream_t st) {
  if (s.bf16) return ffn_e<EltBF16>(s, cpt, x, sel_idx, sel_sig, Wg, Wu, Wd, partial, err, st);
  return ffn_e<EltF32>(s, cpt, x, sel_idx, sel_sig, Wg, Wu, Wd, partial, err, st);
}

template <int C>
cudaError_t reduce_c(const FwdShape &s, int n, int cpt, const float *partial, void *out,
                     ReduceOut kind, cudaStream_t st) {
  const int64_t blocks = (int64_t)((n + C - 1) / C) * s.T;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)blocks), block(kReduceThreads);
  if (kind == ReduceOut::kSplitH)
    return launch_pdl(k_reduce_partials<C, 2>, grid, block, 0, st, partial, out, n, cpt);
  if (kind == ReduceOut::kY && s.bf16)
    return launch_pdl(k_reduce_partials<C, 1>, grid, block, 0, st, partial, out, n, cpt);
  return launch_pdl(k_reduce_partials<C, 0>, grid, block, 0, st, partial, out, n, cpt);
}

cudaError_t launch_reduce_partials(const FwdShape &s, int cpt, const float *partial, void *y,
                                   cudaStream_t st, ReduceOut kind) {
  const int n = (kind == ReduceOut::kSplitH) ? s.r : s.d;
  cudaError_t e;
  if (cpt <= kSmallCpt && n % 4 == 0) {
    const int per_t = (n / 4 + kReduceThreads - 1) / kReduceThreads;
    const int64_t blocks = (int64_t)per_t * s.T;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)blocks), block(kReduceThreads);
    if (kind == ReduceOut::kSplitH)
      e = launch_pdl(k_reduce_few<2>, grid, block, 0, st, partial, y, n, cpt);
    else if (kind == ReduceOut::kY && s.bf16)
      e = launch_pdl(k_reduce_few<1>, grid, block, 0, st, partial, y, n, cpt);
    else
      e = launch_pdl(k_reduce_few<0>, grid, block, 0, st, partial, y, n, cpt);
  } else {
    // many partials: narrow slices and 32 partial groups; else wide slices
    e = cpt >= 32 ? reduce_c<32>(s, n, cpt, partial, y, kind, st)
                  : reduce_c<128>(s, n, cpt, partial, y, kind, st);
  }
  count_launches(1);
  return e;
}

}  // namespace sfn
