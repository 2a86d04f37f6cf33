// decode_fused.cu -- the one-token forward in a single cooperative launch.
//
// The same forward as the few-token kernels ("Continual LLM Upcycling: A
// Predictor-Gated Bank-Wise Sparsity Training Recipe for Dense-to-Sparse
// LLMs", gist.science summary, "1. Architectuur" -- predictor, bank-wise
// hard top-k, sigma(p) in place of the SwiGLU gate -- and "3. Hardware
// Implicaties" -- gate, up and down skip the inactive channels), with the
// four kernels of that path folded into one grid of one CTA per SM:
//
//   phase 0  prologue: the CTA's rows of A go into registers and the rows of
//            B that its banks need are bulk-copied into shared memory, both
//            at once (weights only); x is staged in shared memory.
//   phase 1  h: CTA c computes rows c, c + G, ... of h = A x (one warp per
//            row) and publishes them; grid barrier.
//   phase 2  logits + top-k: CTA c owns the kept slots [s0, s1) of the
//            token (slots are bank-major: slot b*k + q is the q-th kept
//            channel of bank b).  It computes the logits of every bank its
//            slots fall in -- the one or two banks a slot range shares with
//            a neighbour are ranked by both CTAs, identically -- and the
//            banks' top-k words, so it needs nothing from other CTAs.
//   phase 3  the kept rows of its slots stream through a ring of shared-
//            memory stages (1-D bulk copies, evict-first) exactly as in the
//            few-token gate/up/down kernel: a = sigma(p) g u, then the down
//            rows accumulate into registers; one float32 partial row per CTA.
//   phase 4  grid barrier; CTA c sums the G partial rows over its range of
//            y's columns in a fixed order and writes y.
//
// Every sum runs in a fixed order, so results are bit-reproducible.  The two
// grid barriers need every CTA resident: the kernel is launched cooperative
// (the runtime refuses a grid that cannot be co-resident).  The barrier
// state is a pair of counters in device memory shared by all launches on the
// device; cooperative grids of one CTA per SM never run at the same time, and
// the state is back at its resting value after every complete launch.  Every
// wait -- on the barriers and on the ring's mbarriers -- is bounded: on a
// timeout the kernel records kDevErrWaitTimeout, waits (bounded) for its own
// copies in flight and returns; sfn_device_errors(clear) then also resets
// the barrier state.
#include <algorithm>

#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {

namespace {

constexpr int kMaxStagesF = 8;       // ring stages = gate/up warps
constexpr int kDownWarpsF = 8;       // output column eighths
constexpr int kMaxChunksF = 4;       // 16-byte column chunks per down lane
constexpr int kMaxBanksF = 4;        // banks a CTA's slot range may touch
constexpr int kMaxSlotsF = 256;      // kept slots per CTA
constexpr size_t kUnionBudget = 176 * 1024;  // B staging, then the ring
constexpr uint32_t kMaxXBytesF = 16384;
constexpr int kHRowsPerWarpChunk = 16;       // 16-byte loads per lane per pass
constexpr int kRedBatch = 5;                 // partial-row loads in flight per thread

// Grid barrier state: `count` arrivals of the current episode, `gen` the
// number of completed episodes.  Each on its own 128-byte line.
struct GridSync {
  unsigned count;
  unsigned pad0[31];
  unsigned gen;
  unsigned pad1[31];
};
__device__ GridSync g_decode_sync;

struct DecLayout {
  uint32_t row_bytes;
  int stages;
  size_t off_union, off_x, off_h, off_logit, off_key, off_word, off_idx, off_sig, off_a,
      off_bar, off_flag, total;
};

__host__ __device__ constexpr size_t align_to(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline DecLayout dec_layout(int d, int r, int bank, int nb_max) {
  DecLayout L;
  L.row_bytes = (uint32_t)d * 2;
  int s = (int)((kUnionBudget) / (3ull * L.row_bytes));
  L.stages = s < 1 ? 1 : (s > 7 ? 7 : s);
  const size_t ring = (size_t)L.stages * 3 * L.row_bytes;
  const size_t bstage = (size_t)nb_max * bank * r * 2;
  size_t u = ring > bstage ? ring : bstage;
  const size_t red = (size_t)(32 + 4) * 8 * 16;  // reduce staging
  if (red > u) u = red;
  L.off_union = 0;
  L.off_x = align_to(u, 128);
  L.off_h = align_to(L.off_x + L.row_bytes, 128);
  L.off_logit = align_to(L.off_h + (size_t)r * 4, 128);
  L.off_key = L.off_logit + (size_t)kMaxBanksF * 64 * 4;
  L.off_word = L.off_key + (size_t)kMaxBanksF * 64 * 4;
  L.off_idx = L.off_word + (size_t)kMaxBanksF * 8;
  L.off_sig = L.off_idx + (size_t)kMaxSlotsF * 4;
  L.off_a = L.off_sig + (size_t)kMaxSlotsF * 4;
  L.off_bar = align_to(L.off_a + (size_t)kMaxSlotsF * 4, 16);
  L.off_flag = L.off_bar + (5 * kMaxStagesF + 1) * 8;
  L.total = L.off_flag + 16;
  return L;
}

struct DecParams {
  const char *x, *A, *B, *Wg, *Wu, *Wd;
  void *y;          // bf16 [d], or float32 [d] when y_f32
  uint64_t *mask;   // [n_banks] or null
  float *h;         // scratch [r]
  float *partial;   // scratch [G][d]
  int d, d_i, r, bank, k, n_banks, d_s, nb_max;
  bool y_f32;
  unsigned *err;
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier over gridDim.x CTAs (all co-resident).  Writes of every
// thread of the CTA before the call are visible to every thread of every CTA
// after it.  Bounded: false (and kDevErrWaitTimeout) if the other CTAs do not
// arrive in time.
__device__ bool grid_sync(unsigned *err, int *s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned g = ld_acquire_gpu(&g_decode_sync.gen);
    __threadfence();
    const unsigned arrived = atomicAdd(&g_decode_sync.count, 1u);
    if (arrived == gridDim.x - 1) {
      atomicExch(&g_decode_sync.count, 0u);
      __threadfence();
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&g_decode_sync.gen), "r"(g + 1u)
                   : "memory");
    } else {
      const long long t0 = clock64();
      while (ld_acquire_gpu(&g_decode_sync.gen) == g) {
        if (clock64() - t0 > kWaitLimitCycles) {
          report_error(err, kDevErrWaitTimeout);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// blockDim.x = (S + kDownWarpsF + 1) * 32: warps [0, S) gate/up, [S, S + 8)
// down, the last warp produces.  gridDim.x = G CTAs, one per SM.
__global__ void __launch_bounds__((7 + kDownWarpsF + 1) * 32, 1)
    k_decode_fused(const DecParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DecLayout L = dec_layout(p.d, p.r, p.bank, p.nb_max);
  const int S = L.stages;
  const uint32_t row = L.row_bytes;
  unsigned char *uni = smem + L.off_union;
  unsigned char *x_s = smem + L.off_x;
  float *h_s = reinterpret_cast<float *>(smem + L.off_h);
  float *logit_s = reinterpret_cast<float *>(smem + L.off_logit);  // [kMaxBanksF][64]
  uint32_t *key_s = reinterpret_cast<uint32_t *>(smem + L.off_key);
  uint64_t *word_s = reinterpret_cast<uint64_t *>(smem + L.off_word);
  int *idx_s = reinterpret_cast<int *>(smem + L.off_idx);
  float *sig_s = reinterpret_cast<float *>(smem + L.off_sig);
  float *a_s = reinterpret_cast<float *>(smem + L.off_a);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.off_bar);
  uint64_t *gu_full = bar, *gu_empty = bar + kMaxStagesF, *d_full = bar + 2 * kMaxStagesF;
  uint64_t *d_empty = bar + 3 * kMaxStagesF, *a_ready = bar + 4 * kMaxStagesF;
  uint64_t *bbar = bar + 5 * kMaxStagesF;
  int *s_flag = reinterpret_cast<int *>(smem + L.off_flag);

  const int G = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int s0 = (int)(((int64_t)p.d_s * c) / G);
  const int s1 = (int)(((int64_t)p.d_s * (c + 1)) / G);
  const int cnt = s1 - s0;
  const int b_first = s0 / p.k;
  const int nb = cnt > 0 ? (s1 - 1) / p.k - b_first + 1 : 0;
  const uint32_t bbytes = (uint32_t)nb * p.bank * p.r * 2;

  // ---------------------------------------------------------- phase 0
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&gu_full[i], 1);
      mbar_init(&gu_empty[i], 1);
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], kDownWarpsF);
      mbar_init(&a_ready[i], 1);
    }
    mbar_init(bbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && bbytes > 0) {
    // the banks' rows of B are contiguous: one range, in 16 KB pieces
    mbar_arrive_expect_tx(bbar, bbytes);
    const char *src = p.B + (int64_t)b_first * p.bank * p.r * 2;
    for (uint32_t o = 0; o < bbytes; o += 16384) {
      const uint32_t n = bbytes - o < 16384 ? bbytes - o : 16384;
      bulk_g2s(uni + o, src + o, n, bbar);
    }
  }
  // this warp's row of A (row m = c + G * warp), the first pass of its
  // 16-byte loads in flight before x is staged
  const int nchunk = p.d / 8;
  const int m = c + G * warp;
  const bool hrow = warp < nwarps && m < p.r;
  const char *arow = p.A + (int64_t)(hrow ? m : 0) * row;
  uint4 av[kHRowsPerWarpChunk];
#pragma unroll
  for (int u = 0; u < kHRowsPerWarpChunk; ++u) {
    const int q = lane + 32 * u;
    av[u] = (hrow && q < nchunk) ? ld_stream16(arow + (size_t)q * 16) : make_uint4(0, 0, 0, 0);
  }
  pdl_wait();  // x may come from earlier work on the stream
  for (int i = threadIdx.x; i < nchunk; i += blockDim.x)
    *reinterpret_cast<uint4 *>(x_s + (size_t)i * 16) = ld_nc16(p.x + (size_t)i * 16);
  __syncthreads();

  // ---------------------------------------------------------- phase 1: h
  if (hrow) {
    float acc = 0.f;
    for (int q0 = 0; q0 < nchunk; q0 += 32 * kHRowsPerWarpChunk) {
      if (q0 > 0) {
#pragma unroll
        for (int u = 0; u < kHRowsPerWarpChunk; ++u) {
          const int q = q0 + lane + 32 * u;
          av[u] = q < nchunk ? ld_stream16(arow + (size_t)q * 16) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kHRowsPerWarpChunk; ++u) {
        const int q = q0 + lane + 32 * u;
        if (q < nchunk) {
          float a[8], xf[8];
          EltBF16::unpack(av[u], a);
          EltBF16::unpack(*reinterpret_cast<const uint4 *>(x_s + (size_t)q * 16), xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc = fmaf(a[e], xf[e], acc);
        }
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) p.h[m] = acc;
  }
  bool ok = grid_sync(p.err, s_flag);

  // ---------------------------------------------------------- phase 2: logits, top-k
  {
    // B's copies must have landed before anything else, also on the error
    // path (never leave with copies landing)
    const bool landed = bbytes == 0 || mbar_wait(bbar, 0, p.err);
    if (!landed && threadIdx.x == 0) mbar_wait(bbar, 0, p.err);
    ok = __syncthreads_and(ok && landed) != 0;
  }
  if (ok) {
    for (int i = threadIdx.x; i < p.r / 4; i += blockDim.x)
      reinterpret_cast<float4 *>(h_s)[i] = __ldcg(reinterpret_cast<const float4 *>(p.h) + i);
    __syncthreads();
    const int nrows = nb * p.bank;
    const int rchunk = p.r / 8;
    for (int jl0 = warp; jl0 < nrows; jl0 += 4 * nwarps) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c0 = lane; c0 < rchunk; c0 += 64) {
        uint4 v[4][2];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int jl = jl0 + q * nwarps;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int cc = c0 + 32 * u;
            v[q][u] = (jl < nrows && cc < rchunk)
                          ? *reinterpret_cast<const uint4 *>(uni + ((size_t)jl * p.r + (size_t)cc * 8) * 2)
                          : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = c0 + 32 * u;
          if (cc < rchunk) {
            const float4 h0 = *reinterpret_cast<const float4 *>(h_s + cc * 8);
            const float4 h1 = *reinterpret_cast<const float4 *>(h_s + cc * 8 + 4);
            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float w[8];
              EltBF16::unpack(v[q][u], w);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[q] = fmaf(w[e], hv[e], acc[q]);
            }
          }
        }
      }
      // lanes 8q .. 8q + 7 end with row q's sum
      const float v = warp_sum4(acc[0], acc[1], acc[2], acc[3]);
      const int jl = jl0 + (lane >> 3) * nwarps;
      if ((lane & 7) == 0 && jl < nrows) {
        const int bl = jl / p.bank, ch = jl - bl * p.bank;
        logit_s[bl * 64 + ch] = v;
        key_s[bl * 64 + ch] = order_key(v);
      }
    }
    __syncthreads();
    // one warp per bank: the top-k word, then the CTA's slots of that bank
    // in ascending channel order (slot b*k + q = the q-th kept channel)
    for (int bl = warp; bl < nb; bl += nwarps) {
      const int b = b_first + bl;
      const uint64_t word = smem_bank_topk(key_s + bl * 64, p.bank, p.k);
      if (lane == 0) word_s[bl] = word;
      // the CTA holding the bank's first slot writes its mask word
      if (p.mask != nullptr && lane == 0 && b * p.k >= s0 && b * p.k < s1) p.mask[b] = word;
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const int ch = lane + 32 * hlf;
        if (ch < p.bank && ((word >> ch) & 1ull)) {
          const int s = b * p.k + __popcll(word & ((1ull << ch) - 1ull));
          if (s >= s0 && s < s1) {
            idx_s[s - s0] = b * p.bank + ch;
            sig_s[s - s0] = sigmoid_f32(logit_s[bl * 64 + ch]);
          }
        }
      }
    }
    // the B staging area becomes the ring: order the generic-proxy reads of
    // B before the bulk copies that overwrite it
    fence_proxy_async_smem();
    __syncthreads();
  }

  // ---------------------------------------------------------- phase 3: gate/up/down
  unsigned char *gu_ring = uni;                                 // [S][2][row]
  unsigned char *d_ring = uni + (size_t)S * 2 * row;            // [S][row]
  if (ok) {
    if (warp == S + kDownWarpsF) {
      // producer: lane st owns ring stage st
      const int st = lane;
      const uint64_t once = make_evict_first_policy();
      if (st < S) {
        int issued = 0;
        for (int n = st; n < cnt; n += S) {
          const uint32_t use = (uint32_t)(n / S);
          if (use > 0 && (!mbar_wait(&gu_empty[st], (use - 1) & 1u, p.err) ||
                          !mbar_wait(&d_empty[st], (use - 1) & 1u, p.err)))
            break;
          const int64_t j = idx_s[n];
          unsigned char *gdst = gu_ring + (size_t)st * 2 * row;
          mbar_arrive_expect_tx(&gu_full[st], 2 * row);
          bulk_g2s_hint(gdst, p.Wg + j * row, row, &gu_full[st], once);
          bulk_g2s_hint(gdst + row, p.Wu + j * row, row, &gu_full[st], once);
          mbar_arrive_expect_tx(&d_full[st], row);
          bulk_g2s_hint(d_ring + (size_t)st * row, p.Wd + j * row, row, &d_full[st], once);
          issued = use + 1;
        }
        if (issued > 0) {  // never leave while a copy may still be landing
          mbar_wait(&gu_full[st], (uint32_t)(issued - 1) & 1u, p.err);
          mbar_wait(&d_full[st], (uint32_t)(issued - 1) & 1u, p.err);
        }
      }
    } else if (warp < S) {
      // gate / up: a = sigma(p) g u
      const unsigned char *gs = gu_ring + (size_t)warp * 2 * row;
      const unsigned char *us = gs + row;
      for (int n = warp; n < cnt; n += S) {
        if (!mbar_wait(&gu_full[warp], (uint32_t)(n / S) & 1u, p.err)) break;
        float g = 0.f, u = 0.f;
#pragma unroll 4
        for (int q = lane; q < nchunk; q += 32) {
          float wg[8], wu[8], xv[8];
          EltBF16::unpack(*reinterpret_cast<const uint4 *>(gs + (size_t)q * 16), wg);
          EltBF16::unpack(*reinterpret_cast<const uint4 *>(us + (size_t)q * 16), wu);
          EltBF16::unpack(*reinterpret_cast<const uint4 *>(x_s + (size_t)q * 16), xv);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
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
    } else {
      // down: this warp's eighth of the output columns, in registers
      const int dw = warp - S;
      const int nq = nchunk / kDownWarpsF;
      float acc[kMaxChunksF][8];
#pragma unroll
      for (int i = 0; i < kMaxChunksF; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
      for (int n = 0; n < cnt; ++n) {
        const int st = n % S;
        const uint32_t par = (uint32_t)(n / S) & 1u;
        if (!mbar_wait(&d_full[st], par, p.err) || !mbar_wait(&a_ready[st], par, p.err)) break;
        const float a = a_s[n];
        const unsigned char *wr = d_ring + (size_t)st * row + (size_t)dw * nq * 16;
#pragma unroll
        for (int i = 0; i < kMaxChunksF; ++i) {
          const int q = lane + 32 * i;
          if (q < nq) {
            float w[8];
            EltBF16::unpack(*reinterpret_cast<const uint4 *>(wr + (size_t)q * 16), w);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] = fmaf(a, w[e], acc[i][e]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[st]);
      }
      float *out = p.partial + (int64_t)c * p.d + (int64_t)dw * nq * 8;
#pragma unroll
      for (int i = 0; i < kMaxChunksF; ++i) {
        const int q = lane + 32 * i;
        if (q < nq) {
          float4 *dst = reinterpret_cast<float4 *>(out + (size_t)q * 8);
          dst[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
          dst[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
        }
      }
    }
  }
  // every CTA arrives, also one whose earlier wait gave up (so that the
  // others do not wait for it until their own limit)
  const bool ok2 = grid_sync(p.err, s_flag);
  if (!ok || !ok2) return;

  // ---------------------------------------------------------- phase 4: y
  // Quads [q_a, q_b) of y, eight at a time.  Threads (g, qi), g < 32: group g
  // adds partial rows g, g + 32, ... of quad qi (its loads in flight
  // together); then 4 x 8 threads add 8 groups each, then 8 threads the 4
  // parts -- a fixed order throughout.
  const int nq4 = p.d / 4;
  const int q_a = (int)(((int64_t)nq4 * c) / G), q_b = (int)(((int64_t)nq4 * (c + 1)) / G);
  float4 *red = reinterpret_cast<float4 *>(uni);    // [32][8]
  float4 *red2 = red + 32 * 8;                      // [4][8]
  const int qi = threadIdx.x & 7, g = threadIdx.x >> 3;
  auto add4 = [](float4 &a, const float4 &b) {
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  };
  for (int qb0 = q_a; qb0 < q_b; qb0 += 8) {
    const int q = qb0 + qi;
    if (g < 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (q < q_b) {
        const float *src = p.partial + (size_t)q * 4;
        for (int j0 = g; j0 < G; j0 += 32 * kRedBatch) {
          float4 v[kRedBatch];
#pragma unroll
          for (int u = 0; u < kRedBatch; ++u) {
            const int j = j0 + 32 * u;
            v[u] = j < G ? __ldcg(reinterpret_cast<const float4 *>(src + (size_t)j * p.d))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < kRedBatch; ++u) add4(acc, v[u]);
        }
      }
      red[g * 8 + qi] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int part = threadIdx.x >> 3;
      float4 v = red[(part * 8) * 8 + qi];
#pragma unroll
      for (int gg = 1; gg < 8; ++gg) add4(v, red[(part * 8 + gg) * 8 + qi]);
      red2[part * 8 + qi] = v;
    }
    __syncthreads();
    if (threadIdx.x < 8 && q < q_b) {
      float4 v = red2[qi];
#pragma unroll
      for (int part = 1; part < 4; ++part) add4(v, red2[part * 8 + qi]);
      if (p.y_f32) {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.y) + (size_t)q * 4) = v;
      } else {
        uint2 o;
        o.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
        o.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
        *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.y) + (size_t)q * 4) = o;
      }
    }
    __syncthreads();
  }
}

int decode_grid(const DeviceInfo &dev, int plan_sms) {
  return dev.num_sms < plan_sms ? dev.num_sms : plan_sms;
}

// Most banks any CTA's slot range touches, for a grid of G CTAs.
int max_banks_per_cta(const FwdShape &s, int G) {
  int mx = 0;
  for (int c = 0; c < G; ++c) {
    const int s0 = (int)(((int64_t)s.d_s * c) / G), s1 = (int)(((int64_t)s.d_s * (c + 1)) / G);
    if (s1 > s0) mx = std::max(mx, (s1 - 1) / s.k - s0 / s.k + 1);
  }
  return mx;
}

}  // namespace

bool decode_fused_shape_ok(const FwdShape &s, int G) {
  if (!(s.bf16 && s.T == 1 && G >= 1)) return false;
  if (s.d % (8 * kDownWarpsF) != 0 || s.d / 8 / kDownWarpsF > 32 * kMaxChunksF) return false;
  if ((uint32_t)s.d * 2 > kMaxXBytesF || s.r % 8 != 0) return false;
  if ((s.d_s + G - 1) / G > kMaxSlotsF) return false;
  const int nbm = max_banks_per_cta(s, G);
  if (nbm > kMaxBanksF) return false;
  if ((size_t)nbm * s.bank * s.r * 2 > kUnionBudget) return false;
  // the h phase: rows c + G * warp need ceil(r / G) warps
  const DecLayout L = dec_layout(s.d, s.r, s.bank, nbm);
  const int nwarps = L.stages + kDownWarpsF + 1;
  if ((s.r + G - 1) / G > nwarps) return false;
  return L.total <= 227 * 1024;
}

size_t decode_fused_scratch(const FwdShape &s, int G) {
  return align_up((size_t)s.r * 4, 256) + (size_t)G * s.d * 4;
}

cudaError_t launch_decode_fused(const FwdShape &s, const DeviceInfo &dev, int plan_sms,
                                const void *x, const void *A, const void *B, const void *Wg,
                                const void *Wu, const void *Wd, void *y, bool y_f32,
                                uint64_t *mask, void *scratch, cudaStream_t st) {
  const int G = decode_grid(dev, plan_sms);
  if (!decode_fused_shape_ok(s, G)) return cudaErrorInvalidValue;
  const int nbm = max_banks_per_cta(s, G);
  const DecLayout L = dec_layout(s.d, s.r, s.bank, nbm);
  const int threads = (L.stages + kDownWarpsF + 1) * 32;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(k_decode_fused), L.total);
  if (e != cudaSuccess) return e;
  DecParams p{};
  p.x = static_cast<const char *>(x);
  p.A = static_cast<const char *>(A);
  p.B = static_cast<const char *>(B);
  p.Wg = static_cast<const char *>(Wg);
  p.Wu = static_cast<const char *>(Wu);
  p.Wd = static_cast<const char *>(Wd);
  p.y = y;
  p.y_f32 = y_f32;
  p.mask = mask;
  p.h = static_cast<float *>(scratch);
  p.partial = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                        align_up((size_t)s.r * 4, 256));
  p.d = s.d;
  p.d_i = s.d_i;
  p.r = s.r;
  p.bank = s.bank;
  p.k = s.k;
  p.n_banks = s.n_banks;
  p.d_s = s.d_s;
  p.nb_max = nbm;
  p.err = dev.err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_decode_fused, p);
  count_launches(1);
  return e;
}

cudaError_t reset_decode_sync() {
  void *addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, g_decode_sync);
  if (e != cudaSuccess) return e;
  return cudaMemset(addr, 0, sizeof(GridSync));
}

}  // namespace sfn
