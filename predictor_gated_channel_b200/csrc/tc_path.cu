// tc_path.cu -- the many-token path on the 5th-generation tensor cores.
//
// The same forward as the few-token path ("Continual LLM Upcycling: A
// Predictor-Gated Bank-Wise Sparsity Training Recipe for Dense-to-Sparse
// LLMs", gist.science summary, "1. Architectuur" and "3. Hardware
// Implicaties"), computed as four tiled contractions over 128-token tiles:
//
//   G1  H = X A^T                    -> H split into bf16 hi + lo halves
//   G2  P = H_hi B^T + H_lo B^T      -> bank top-k fused into the epilogue:
//                                       mask words + sigma(p) of kept channels
//                                       (or the raw fp32 logits)
//   G3  [G | U] = X [W_gate; W_up]^T -> a = sigma(p) g u on kept channels, 0
//                                       elsewhere (bf16, [T][d_i])
//   G4  Y = A_act W_down             -> y (bf16)
//
// Splitting h = hi + lo keeps the logits fp32-accurate (about 2^-16 relative)
// although the tensor cores take bf16 operands: B is exactly bf16, so only
// the error of h - hi - lo (about 2^-17 |h|) remains.
//
// Each GEMM is one persistent, warp-specialised kernel (one CTA per SM):
//   warp 0      TMA producer: tiled loads (128-byte swizzle, no multicast)
//               into a ring of shared-memory stages
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M 128, N <= 256, K 16, bf16 -> f32) into one of two TMEM
//               accumulators and commits stage releases / tile completions
//   warps 2..   epilogue (4 warps for G1, 8 for G2-G4: two per TMEM lane
//               quadrant, splitting a tile's banks or column chunks):
//               tcgen05.ld of the warp's 32 TMEM lanes (= 32 token rows), the
//               epilogue arithmetic, global stores; they release the
//               accumulator so the next tile's MMAs overlap this epilogue
// With one token tile every weight byte is read once: the weight loads then
// carry an evict-first L2 policy, and the producer issues the first stages'
// weight loads before its dependency wait.  There, G2 also runs inside G3
// (k_tc_logits_gateup, below).  With few token tiles, G1 and G4 split K over
// the SMs into ranges that differ by at most one block, and write float32
// partials that a separate kernel sums in a fixed order.
// The same engine runs the Dense-4x comparison's gate/up GEMM and the
// backward's float32-output contractions (A and B K-major or MN-major).
// Every mbarrier wait is bounded (async_util.cuh).
#include <cudaTypedefs.h>

#include <algorithm>

#include <initializer_list>
#include <mutex>
#include <type_traits>

#include "sfn_internal.cuh"
#include "tc_util.cuh"

namespace sfn {

// ------------------------------------------------------------------ tensor maps
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// Row-major bf16 matrix [outer][inner] with rows `stride` elements apart
// (0: inner), box {box_inner, box_outer}, 128-byte swizzle, zero fill
// outside.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer, uint64_t stride) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {(stride ? stride : inner) * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

constexpr int kBM = 128;                       // token rows per tile (UMMA M)
constexpr int kBK = 64;                        // K per stage: 128-byte rows
constexpr uint32_t kTileA = kBM * kBK * 2;     // 16 KB

constexpr int kAccCols = 256;                  // TMEM columns per accumulator
constexpr size_t kMaxDynSmem = 232448;            // 227 KB per CTA on sm_100
constexpr int kGroupM = 8;                     // tile rasterisation group

enum : int {
  kEpiHSplit = 0,
  kEpiLogits = 1,
  kEpiTopk = 2,
  kEpiGateUp = 3,
  kEpiDown = 4,
  kEpiDense4x = 5,  // gate/up GEMM of the post-hoc amplitude top-k comparison
  // plain float32 products C (=, +=) A B of the backward; the suffix gives
  // the storage of A and B: K = K-major ([M][K], [N][K]), M = MN-major
  // ([K][M], [K][N])
  kEpiF32KK = 6,
  kEpiF32KM = 7,
  kEpiF32MM = 8
};

struct TcParams {
  int64_t T;
  int tiles_m, tiles_n, k_blocks;
  int ksplit;             // K ranges per output tile (>1: fp32 partial outputs)
  int bn;                 // UMMA N
  int stages;
  uint32_t stage_bytes;   // bytes delivered per stage (A tiles + B)
  uint32_t idesc;
  void *out;              // H2 / logits / a_act / y
  uint64_t *mask;         // top-k: written; gate/up: read
  float *sig;             // top-k: written; gate/up: read  ([T][n_banks][k])
  int ld_out;             // elements per output row
  int r, k, n_banks;
  bool f32_out;           // down: float32 y (no bf16 rounding), ksplit == 1
  int a_rows;             // token rows the TMA loads per A tile (<= kBM; 0: kBM).  With
                          // fewer tokens than a tile, rows past them are not loaded: the
                          // MMA reads stale shared memory there, which only reaches
                          // accumulator rows the epilogue never stores
  uint32_t tx_bytes;      // bytes the TMA delivers per stage
  uint32_t a_tile_bytes;  // bytes of one A tile in a stage (a_rows x 128)
  float *tau;             // top-k, if set: threshold per (token, bank) and float32 logits
                          // into out ([T][ld_out]); sig may then be null
  bool b_once;            // the B operand (weights) is read once (one token tile): its
                          // loads carry an evict-first L2 policy
  bool accumulate;        // float32 products: add to the output instead of overwriting
  int n_valid;            // float32 products: output columns (the last N tile may run
                          // past them: its loads zero-fill, its stores skip them)
  unsigned *err;
};

template <int kEpi>
struct EpiTraits {
  static constexpr int kNumA = (kEpi == kEpiLogits || kEpi == kEpiTopk) ? 2 : 1;
  static constexpr bool kF32 = (kEpi == kEpiF32KK || kEpi == kEpiF32KM || kEpi == kEpiF32MM);
  static constexpr bool kAMnMajor = (kEpi == kEpiF32MM);
  static constexpr bool kBMnMajor = (kEpi == kEpiDown || kEpi == kEpiF32KM || kEpi == kEpiF32MM);
  static constexpr bool kGateUpB = (kEpi == kEpiGateUp || kEpi == kEpiDense4x);
  // epilogue warps: two per TMEM lane quadrant for the top-k (its sorting
  // networks, not the MMAs, bound that GEMM) and for gate/up and down (with
  // one tile per CTA at few tokens, their epilogue is a serial tail after
  // the mainloop), splitting the tile's banks or column chunks
  static constexpr int kEpiWarps =
      (kEpi == kEpiTopk || kEpi == kEpiGateUp || kEpi == kEpiDown || kF32) ? 8 : 4;
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
};

__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int &mb,
                                            int &nb) {
  const int group = tile / (kGroupM * tiles_n);
  const int first_m = group * kGroupM;
  const int gm = min(kGroupM, tiles_m - first_m);
  const int idx = tile - group * kGroupM * tiles_n;
  mb = first_m + idx % gm;
  nb = idx / gm;
}

// Work unit -> output tile and its K-block range [kb0, kb1).  The K splits
// differ in length by at most one block, so none is empty while ksplit <=
// k_blocks (equal ceil-sized ranges would leave the last splits empty when
// ksplit does not divide k_blocks).
__device__ __forceinline__ void unit_coords(int unit, const TcParams &p, int &mb, int &nb,
                                            int &kb0, int &kb1) {
  const int split = unit % p.ksplit;
  tile_coords(unit / p.ksplit, p.tiles_m, p.tiles_n, mb, nb);
  kb0 = (int)((int64_t)p.k_blocks * split / p.ksplit);
  kb1 = (int)((int64_t)p.k_blocks * (split + 1) / p.ksplit);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
}

// s[A..A+16) and s[B..B+16) sorted descending -> s[A..A+16) = the 16 largest
// of both, sorted descending (max with the reversed other list gives a
// bitonic sequence, which a half-cleaner cascade sorts).
template <int A, int B>
__device__ __forceinline__ void merge_top16(uint32_t (&s)[64]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) s[A + i] = max(s[A + i], s[B + 15 - i]);
#pragma unroll
  for (int stride = 8; stride > 0; stride >>= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if ((i & stride) == 0) cex_desc(s[A + i], s[A + i + stride]);
}

// Logistic function for the tensor-core epilogues (hardware exp2 and
// reciprocal; relative error far below the bf16 rounding of the values it
// scales).  Saturates to exactly 0 and 1.
__device__ __forceinline__ float sigmoid_fast(float z) {
  return __fdividef(1.0f, 1.0f + __expf(-z));
}


// k-th largest of 64 order keys (s is reordered), and the number of keys
// strictly above it.
__device__ __forceinline__ void keys_threshold(uint32_t (&s)[64], int k, uint32_t &tau, int &gt) {
  gt = 0;
  if (k == 16) {
    BitonicSort<0, 16, 2>::run(s);
    BitonicSort<16, 16, 2>::run(s);
    BitonicSort<32, 16, 2>::run(s);
    BitonicSort<48, 16, 2>::run(s);
    merge_top16<0, 16>(s);
    merge_top16<32, 48>(s);
    tau = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < 16; ++i) tau = min(tau, max(s[i], s[47 - i]));
#pragma unroll
    for (int i = 0; i < 16; ++i) gt += max(s[i], s[47 - i]) > tau;
  } else {
    BitonicSort<0, 64, 2>::run(s);
    tau = s[0];
#pragma unroll
    for (int i = 1; i < 64; ++i) tau = (i == k - 1) ? s[i] : tau;
#pragma unroll
    for (int i = 0; i < 64; ++i) gt += s[i] > tau;
  }
}

// k-th largest order key of the 64 logits held in TMEM columns
// [taddr, taddr + 64) of this thread's row, and the number of keys strictly
// above it.
__device__ __forceinline__ void bank_threshold(uint32_t taddr, int k, uint32_t &tau, int &gt) {
  if (k >= 64) {  // k = bank: every channel kept (key >= 0 = tau), no ranking
    tau = 0u;
    gt = 0;
    return;
  }
  if (k <= 16) {
    // A running list of the 16 largest keys, sorted descending, merged with
    // each sorted group of 16 in turn.  A loop, not unrolled: the straight-line
    // version of this epilogue was long enough to stall on instruction fetch.
    // Keys are >= 0, so starting from zeros the first merge takes group 0 as is.
    uint32_t top[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) top[i] = 0u;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      uint32_t r[16];
      tmem_ld_32x32b_x16(taddr + g * 16, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = order_key(__uint_as_float(r[i]));
      BitonicSort<0, 16, 2>::run(r);
#pragma unroll
      for (int i = 0; i < 16; ++i) top[i] = max(top[i], r[15 - i]);
#pragma unroll
      for (int stride = 8; stride > 0; stride >>= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if ((i & stride) == 0) cex_desc(top[i], top[i + stride]);
    }
    tau = top[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) tau = (i == k - 1) ? top[i] : tau;
    gt = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) gt += top[i] > tau;
    return;
  }
  // k > 16: sort all 64 keys
  uint32_t s[64];
  tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
  tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 64; ++i) s[i] = order_key(__uint_as_float(s[i]));
  BitonicSort<0, 64, 2>::run(s);
  tau = s[0];
#pragma unroll
  for (int i = 1; i < 64; ++i) tau = (i == k - 1) ? s[i] : tau;
  gt = 0;
#pragma unroll
  for (int i = 0; i < 64; ++i) gt += s[i] > tau;
}

template <int kEpi>
__global__ void __launch_bounds__(EpiTraits<kEpi>::kThreads, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
              const __grid_constant__ CUtensorMap tB2, const TcParams p) {
  using Tr = EpiTraits<kEpi>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * p.stage_bytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + p.stages;
  uint64_t *tfull = bars + 2 * p.stages;
  uint64_t *tempty = tfull + 2;
  uint64_t *done = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  // epilogue staging rows (top-k: kept logits of one bank per thread row)
  float *stage_rows_smem = reinterpret_cast<float *>(smem + (size_t)p.stages * p.stage_bytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.tiles_m * p.tiles_n * p.ksplit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], Tr::kEpiWarps * 32);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * kAccCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Operands may come from earlier work on the stream.  The producer waits
  // later: the weights (every GEMM's B operand) are not written by earlier
  // work, so with one token tile it issues the first stages' weight loads
  // before its wait.
  if (!p.b_once || warp != 0) {
    pdl_wait();
    pdl_launch_dependents();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tA);
      prefetch_tmap(&tB);
      if (Tr::kGateUpB) prefetch_tmap(&tB2);
      // Two versions of the loop, chosen once: kOnce (one token tile,
      // weights read once) loads the weights with an evict-first L2 policy
      // and issues the first stages' weights before the dependency wait;
      // otherwise the loop is the plain one (a runtime test per load cost
      // the down GEMM about 6 % at 4096 tokens).
      auto produce = [&](auto once_tag) {
        constexpr bool kOnce = decltype(once_tag)::value;
        uint32_t it = 0;
        bool ok = true;
        const uint64_t once = kOnce ? make_evict_first_policy() : 0ull;
        auto load_b = [&](void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
          if constexpr (kOnce)
            tma_load_2d_hint(dst, map, c0, c1, bar, once);
          else
            tma_load_2d(dst, map, c0, c1, bar);
        };
        // the weights of stage s for K block kb and N tile nb
        auto issue_b = [&](int s, int kb, int nb) {
          unsigned char *b = smem + (size_t)s * p.stage_bytes + Tr::kNumA * p.a_tile_bytes;
          if (Tr::kGateUpB) {
            load_b(b, &tB, kb * kBK, nb * (p.bn / 2), &full[s]);
            load_b(b + (p.bn / 2) * 128, &tB2, kb * kBK, nb * (p.bn / 2), &full[s]);
          } else if (kEpi == kEpiDown) {
            // [K][N] storage: four boxes of 64 N-elements x 64 K-rows (N 256).
            // Kept as a fixed, unrolled loop: a runtime bound here (bn / 64 boxes)
            // or a guard on it cost the down GEMM 9-16 % at prefill.
#pragma unroll
            for (int q = 0; q < 4; ++q)
              load_b(b + q * 8192, &tB, nb * kAccCols + q * 64, kb * kBK, &full[s]);
          } else if (Tr::kBMnMajor) {
            // float32 products, [K][N] storage: bn/64 boxes of 64 x 64
            for (int q = 0; q < p.bn / 64; ++q)
              load_b(b + q * 8192, &tB, nb * p.bn + q * 64, kb * kBK, &full[s]);
          } else {
            load_b(b, &tB, kb * kBK, nb * p.bn, &full[s]);
          }
        };
        // kOnce: before the wait, the weights of the first unit's first stages
        int pre = 0;
        if constexpr (kOnce) {
          if ((int)blockIdx.x < total) {
            int mb, nb, kb0, kb1;
            unit_coords(blockIdx.x, p, mb, nb, kb0, kb1);
            pre = max(0, min(p.stages, kb1 - kb0));
            for (int j = 0; j < pre; ++j) {
              mbar_arrive_expect_tx(&full[j], p.tx_bytes);
              issue_b(j, kb0 + j, nb);
            }
          }
          pdl_wait();
          pdl_launch_dependents();
        }
        for (int unit = blockIdx.x; unit < total && ok; unit += gridDim.x) {
          int mb, nb, kb0, kb1;
          unit_coords(unit, p, mb, nb, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = (int)(it % p.stages);
            const uint32_t use = it / p.stages;
            if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1u, p.err)) {
              ok = false;
              break;
            }
            unsigned char *a = smem + (size_t)s * p.stage_bytes;
            const bool fresh = !kOnce || (int)it >= pre;  // weights not issued yet
            if (fresh) mbar_arrive_expect_tx(&full[s], p.tx_bytes);
            if (Tr::kAMnMajor) {
              // [K][M] storage: two boxes of 64 M-elements x 64 K-rows
              tma_load_2d(a, &tA, mb * kBM, kb * kBK, &full[s]);
              tma_load_2d(a + 8192, &tA, mb * kBM + 64, kb * kBK, &full[s]);
            } else {
              tma_load_2d(a, &tA, kb * kBK, mb * kBM, &full[s]);
            }
            if (Tr::kNumA == 2)
              tma_load_2d(a + p.a_tile_bytes, &tA, p.r + kb * kBK, mb * kBM, &full[s]);
            if (fresh) issue_b(s, kb, nb);
          }
        }
        // wait (bounded) until the last load of every stage has landed (a
        // stage whose weights went out before the wait counts as issued)
        const uint32_t issued = it > (uint32_t)pre ? it : (uint32_t)pre;
        for (int s = 0; s < p.stages && (uint32_t)s < issued; ++s) {
          const uint32_t last = s + ((issued - 1 - s) / p.stages) * p.stages;
          mbar_wait(&full[s], (last / p.stages) & 1u, p.err);
        }
      };
      if (p.b_once)
        produce(std::true_type{});
      else
        produce(std::false_type{});
    } else if (p.b_once) {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < total && ok; unit += gridDim.x, ++lt) {
        int mb, nb, kb0, kb1;
        unit_coords(unit, p, mb, nb, kb0, kb1);
        const uint32_t acc = lt & 1u, use = lt >> 1;
        if (use > 0 && !mbar_wait(&tempty[acc], (use - 1) & 1u, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = (int)(it % p.stages);
          if (!mbar_wait(&full[s], (it / p.stages) & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const unsigned char *a = smem + (size_t)s * p.stage_bytes;
          const unsigned char *b = a + Tr::kNumA * p.a_tile_bytes;
          const uint64_t adesc =
              Tr::kAMnMajor ? desc_mnmajor_sw128(a, 8192) : desc_kmajor_sw128(a);
          const uint64_t adesc2 = desc_kmajor_sw128(a + p.a_tile_bytes);
          const uint64_t bdesc =
              Tr::kBMnMajor ? desc_mnmajor_sw128(b, 8192) : desc_kmajor_sw128(b);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // along K: 16 elements = 32 bytes (K-major) or 16 rows of 128
            // bytes (MN-major), in units of 16 bytes
            const uint64_t aoff = Tr::kAMnMajor ? (uint64_t)(kk * 2048 >> 4) : (uint64_t)(kk * 2);
            const uint64_t boff = Tr::kBMnMajor ? (uint64_t)(kk * 2048 >> 4) : (uint64_t)(kk * 2);
            umma_f16(d_tmem, adesc + aoff, bdesc + boff, p.idesc,
                     (kb > kb0 || kk > 0) ? 1u : 0u);
            if (Tr::kNumA == 2) umma_f16(d_tmem, adesc2 + (uint64_t)(kk * 2), bdesc + boff, p.idesc, 1u);
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // all MMAs of this CTA complete before TMEM is released
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;    // token row inside the tile
    const int half_id = (warp - 2) >> 2;  // which of a quadrant's epilogue warps
    uint32_t lt = 0;
    for (int unit = blockIdx.x; unit < total; unit += gridDim.x, ++lt) {
      int mb, nb, kb0, kb1;
      unit_coords(unit, p, mb, nb, kb0, kb1);
      const uint32_t acc = lt & 1u, use = lt >> 1;
      if (!mbar_wait(&tfull[acc], use & 1u, p.err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * kAccCols;
      const int64_t t = (int64_t)mb * kBM + row;
      const bool valid = t < p.T;

      if (kEpi == kEpiHSplit && p.ksplit == 1) {
        uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
        for (int c0 = 0; c0 < p.bn; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c0, v);
          tmem_ld_wait();
          if (valid) {
            const int col = nb * p.bn + c0;
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float f0 = __uint_as_float(v[i]), f1 = __uint_as_float(v[i + 1]);
              const uint16_t h0 = f32_to_bf16_bits(f0), h1 = f32_to_bf16_bits(f1);
              const float r0 = f0 - __uint_as_float((uint32_t)h0 << 16);
              const float r1 = f1 - __uint_as_float((uint32_t)h1 << 16);
              hi[i / 2] = (uint32_t)h0 | ((uint32_t)h1 << 16);
              lo[i / 2] = pack_bf16x2(r0, r1);
            }
            uint4 *dh = reinterpret_cast<uint4 *>(out + t * p.ld_out + col);
            uint4 *dl = reinterpret_cast<uint4 *>(out + t * p.ld_out + p.r + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dh[i] = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
              dl[i] = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
            }
          }
        }
      } else if (kEpi == kEpiLogits || kEpi == kEpiDown || kEpi == kEpiHSplit || Tr::kF32) {
        for (int c0 = 32 * half_id; c0 < p.bn; c0 += 32 * (Tr::kEpiWarps / 4)) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c0, v);
          tmem_ld_wait();
          if (valid && Tr::kF32 && nb * p.bn + c0 < p.n_valid) {
            // C (=, +=) A B, float32 [M][ld_out]
            float *dst = reinterpret_cast<float *>(p.out) + t * p.ld_out + nb * p.bn + c0;
            if (p.accumulate) {
              float4 o[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) o[i] = reinterpret_cast<const float4 *>(dst)[i];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                o[i].x += __uint_as_float(v[4 * i]);
                o[i].y += __uint_as_float(v[4 * i + 1]);
                o[i].z += __uint_as_float(v[4 * i + 2]);
                o[i].w += __uint_as_float(v[4 * i + 3]);
                reinterpret_cast<float4 *>(dst)[i] = o[i];
              }
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                reinterpret_cast<uint4 *>(dst)[i] =
                    make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          } else if (valid && !Tr::kF32) {
            const int col = nb * p.bn + c0;
            if (kEpi != kEpiDown || p.ksplit > 1 || p.f32_out) {
              // fp32 logits, or fp32 partial sums [T][ksplit][ld_out]
              const int64_t orow = (p.ksplit > 1) ? t * p.ksplit + unit % p.ksplit : t;
              uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<float *>(p.out) +
                                                     orow * p.ld_out + col);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
              uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) +
                                                     t * p.ld_out + col);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dst[i] = make_uint4(
                    pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
              }
            }
          }
        }
      } else if (kEpi == kEpiTopk) {
        // bn/64 banks of 64 channels per tile.  The mask pass is branch-free: the
        // logits of kept channels are compacted, in channel order, into this
        // thread's staging row; sigma is then evaluated for those k only.
        const int srow = p.k | 1;  // staged floats per thread row (odd: no bank conflicts)
        float *stg = stage_rows_smem + (half_id * kBM + row) * srow;
        const int banks_per_tile = p.bn / 64;
        for (int bl = half_id; bl < banks_per_tile; bl += Tr::kEpiWarps / 4) {
          uint32_t tau;
          int gt;
          bank_threshold(taddr + bl * 64, p.k, tau, gt);
          const int need = p.k - gt;
          const int bank = nb * banks_per_tile + bl;
          int eq = 0, cnt = 0;
          uint64_t word = 0ull;
          uint32_t rest = 0u;  // rest: largest key not kept
          // four groups of 16 channels, as a loop (code size, as above)
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(taddr + bl * 64 + g * 16, v);
            tmem_ld_wait();
            if (p.tau != nullptr && valid) {
              uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<float *>(p.out) +
                                                     t * p.ld_out + bank * 64 + g * 16);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            uint32_t b = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t key = order_key(__uint_as_float(v[i]));
              const bool take = (key > tau) | ((key == tau) & (eq < need));
              eq += (key == tau);
              b |= (uint32_t)take << i;
              rest = max(rest, take ? 0u : key);
              if (take) stg[cnt] = __uint_as_float(v[i]);
              cnt += take;
            }
            word |= (uint64_t)b << (g * 16);
          }
          if (valid && p.tau != nullptr)
            p.tau[t * p.n_banks + bank] = (p.k < 64)
                                              ? 0.5f * (key_value(tau) + key_value(rest))
                                              : __int_as_float(0x7fc00000);
          if (valid) p.mask[t * p.n_banks + bank] = word;
          if (valid && p.sig != nullptr) {
            float *sig_out = p.sig + (t * p.n_banks + bank) * (int64_t)p.k;
            if ((p.k & 3) == 0) {
              for (int s4 = 0; s4 < p.k; s4 += 4)
                *reinterpret_cast<float4 *>(sig_out + s4) =
                    make_float4(sigmoid_fast(stg[s4]), sigmoid_fast(stg[s4 + 1]),
                                sigmoid_fast(stg[s4 + 2]), sigmoid_fast(stg[s4 + 3]));
            } else {
              for (int s1 = 0; s1 < p.k; ++s1) sig_out[s1] = sigmoid_fast(stg[s1]);
            }
          }
        }
      } else if (kEpi == kEpiGateUp) {
        // channels nb*bn/2 .. +bn/2-1 (bn/128 banks); accumulator columns
        // [0, bn/2) hold g, [bn/2, bn) hold u
        uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
        const int half_n = p.bn / 2;
        for (int h = half_id; h < half_n / 64; h += Tr::kEpiWarps / 4) {
          const int bank = nb * (half_n / 64) + h;
          const uint64_t word = valid ? p.mask[t * p.n_banks + bank] : 0ull;
          const float *sig_in = p.sig + (t * p.n_banks + bank) * (int64_t)p.k;
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(taddr + h * 64 + c0, g);
            tmem_ld_32x32b_x32(taddr + half_n + h * 64 + c0, u);
            tmem_ld_wait();
            if (valid) {
              uint32_t packed[16];
              int rank = __popcll(word & ((1ull << c0) - 1ull));
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                float a2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const bool on = (word >> (c0 + i + e)) & 1ull;
                  const float sg = on ? sig_in[rank] : 0.f;
                  a2[e] = on ? sg * __uint_as_float(g[i + e]) * __uint_as_float(u[i + e]) : 0.f;
                  rank += on;
                }
                packed[i / 2] = pack_bf16x2(a2[0], a2[1]);
              }
              uint4 *dst = reinterpret_cast<uint4 *>(out + t * p.ld_out + bank * 64 + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                    packed[4 * i + 3]);
            }
          }
        }
      }
      if (kEpi == kEpiDense4x) {
        // act = silu(g) u for every channel; per bank keep the k largest
        // |act| (ties to the lower channel), zero the rest; bf16 out
        uint16_t *out = reinterpret_cast<uint16_t *>(p.out);
        const int half_n = p.bn / 2;
        for (int h = 0; h < half_n / 64; ++h) {
          const int bank = nb * (half_n / 64) + h;
          // pass 1: order keys of |act| for the 64 channels, then the threshold
          uint32_t keys[64];
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(taddr + h * 64 + c0, g);
            tmem_ld_32x32b_x32(taddr + half_n + h * 64 + c0, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float gv = __uint_as_float(g[i]);
              keys[c0 + i] = order_key(fabsf(gv * sigmoid_fast(gv) * __uint_as_float(u[i])));
            }
          }
          uint32_t tau;
          int gt;
          keys_threshold(keys, p.k, tau, gt);
          const int need = p.k - gt;
          int eq = 0;
          uint32_t bits[2] = {0u, 0u};
          // pass 2: recompute act half a bank at a time, keep or zero, store
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(taddr + h * 64 + c0, g);
            tmem_ld_32x32b_x32(taddr + half_n + h * 64 + c0, u);
            tmem_ld_wait();
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float o2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float gv = __uint_as_float(g[i + e]);
                const float a = gv * sigmoid_fast(gv) * __uint_as_float(u[i + e]);
                const uint32_t key = order_key(fabsf(a));
                const bool take = (key > tau) | ((key == tau) & (eq < need));
                eq += (key == tau);
                bits[c0 >> 5] |= (uint32_t)take << (i + e);
                o2[e] = take ? a : 0.f;
              }
              packed[i / 2] = pack_bf16x2(o2[0], o2[1]);
            }
            if (valid) {
              uint4 *dst = reinterpret_cast<uint4 *>(out + t * p.ld_out + bank * 64 + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                    packed[4 * i + 3]);
            }
          }
          if (valid) p.mask[t * p.n_banks + bank] = ((uint64_t)bits[1] << 32) | bits[0];
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

// ------------------------------------------------------- one token tile: G2 + G3
// With all tokens in one tile, the logits GEMM (G2) is folded into the
// gate/up GEMM (G3): a unit is 128 channels (two banks), and its K sequence
// is first the r/64 logits blocks (A = H hi and H lo, B = the banks' rows of
// B), then the d/64 gate/up blocks (A = x, B = the channels' W_gate and
// W_up rows).  The logits accumulator (TMEM columns [256, 384)) completes
// early; the epilogue ranks the two banks from it while the MMA warp goes on
// with the gate/up blocks, and keeps each row's mask word and the kept
// channels' sigma for the gate/up epilogue of the same (row, bank) -- the same
// thread, so nothing crosses warps.  The separate logits kernel, its ramp and
// its top-k tail disappear; the top-k work overlaps the weight stream.
struct G23Params {
  int64_t T;
  int n_units;            // d_i / 128
  int kb_l, kb_gu;        // logits blocks (r / 64), gate/up blocks (d / 64)
  int stages;
  uint32_t stage_bytes, a_tile_bytes, tx_l, tx_gu;
  uint32_t idesc_l, idesc_gu;
  int r, k, n_banks, ld_out;
  uint16_t *act;          // [T][d_i] bf16
  uint64_t *mask;         // [T][n_banks], or null
  unsigned *err;
};

constexpr int kG23EpiWarps = 8;
constexpr int kG23Threads = (2 + kG23EpiWarps) * 32;

__global__ void __launch_bounds__(kG23Threads, 1)
    k_tc_logits_gateup(const __grid_constant__ CUtensorMap tH,
                       const __grid_constant__ CUtensorMap tBw,
                       const __grid_constant__ CUtensorMap tX,
                       const __grid_constant__ CUtensorMap tG,
                       const __grid_constant__ CUtensorMap tU, const G23Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * p.stage_bytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + p.stages;
  uint64_t *lfull = bars + 2 * p.stages, *lempty = lfull + 1;
  uint64_t *gfull = lfull + 2, *gempty = lfull + 3;
  uint64_t *done = lfull + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  float *stage_rows = reinterpret_cast<float *>(smem + (size_t)p.stages * p.stage_bytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = p.kb_l + p.kb_gu;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(lfull, 1);
    mbar_init(lempty, kG23EpiWarps * 32);
    mbar_init(gfull, 1);
    mbar_init(gempty, kG23EpiWarps * 32);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * kAccCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (warp != 0) {
    pdl_wait();
    pdl_launch_dependents();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tH);
      prefetch_tmap(&tBw);
      prefetch_tmap(&tX);
      prefetch_tmap(&tG);
      prefetch_tmap(&tU);
      // every weight byte is read once: evict-first
      const uint64_t once = make_evict_first_policy();
      auto issue_w = [&](int s, int i, int nb) {  // weights of block i
        unsigned char *st = smem + (size_t)s * p.stage_bytes;
        if (i < p.kb_l) {
          tma_load_2d_hint(st + 2 * p.a_tile_bytes, &tBw, i * kBK, nb * 128, &full[s], once);
        } else {
          const int kb = i - p.kb_l;
          tma_load_2d_hint(st + p.a_tile_bytes, &tG, kb * kBK, nb * 128, &full[s], once);
          tma_load_2d_hint(st + p.a_tile_bytes + 16384, &tU, kb * kBK, nb * 128, &full[s], once);
        }
      };
      auto issue_t = [&](int s, int i) {  // token operand of block i
        unsigned char *st = smem + (size_t)s * p.stage_bytes;
        if (i < p.kb_l) {
          tma_load_2d(st, &tH, i * kBK, 0, &full[s]);
          tma_load_2d(st + p.a_tile_bytes, &tH, p.r + i * kBK, 0, &full[s]);
        } else {
          tma_load_2d(st, &tX, (i - p.kb_l) * kBK, 0, &full[s]);
        }
      };
      // before the dependency wait: the first unit's first stages' weights
      int pre = 0;
      if ((int)blockIdx.x < p.n_units) {
        pre = min(p.stages, nblk);
        for (int j = 0; j < pre; ++j) {
          mbar_arrive_expect_tx(&full[j], j < p.kb_l ? p.tx_l : p.tx_gu);
          issue_w(j, j, blockIdx.x);
        }
      }
      pdl_wait();
      pdl_launch_dependents();
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.n_units && ok; unit += gridDim.x) {
        for (int i = 0; i < nblk; ++i, ++it) {
          const int s = (int)(it % p.stages);
          const uint32_t use = it / p.stages;
          if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1u, p.err)) {
            ok = false;
            break;
          }
          if ((int)it >= pre) {
            mbar_arrive_expect_tx(&full[s], i < p.kb_l ? p.tx_l : p.tx_gu);
            issue_w(s, i, unit);
          }
          issue_t(s, i);
        }
      }
      const uint32_t issued = it > (uint32_t)pre ? it : (uint32_t)pre;
      for (int s = 0; s < p.stages && (uint32_t)s < issued; ++s) {
        const uint32_t last = s + ((issued - 1 - s) / p.stages) * p.stages;
        mbar_wait(&full[s], (last / p.stages) & 1u, p.err);
      }
    } else {
      pdl_wait();
      pdl_launch_dependents();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t d_gu = tmem_base, d_l = tmem_base + kAccCols;
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.n_units && ok; unit += gridDim.x, ++lt) {
        for (int i = 0; i < nblk; ++i, ++it) {
          // single accumulators: before a unit's first logits (gate/up) MMA,
          // the previous unit's epilogue must have read them
          if (lt > 0 && i == 0 && !mbar_wait(lempty, (lt - 1) & 1u, p.err)) ok = false;
          if (lt > 0 && i == p.kb_l && !mbar_wait(gempty, (lt - 1) & 1u, p.err)) ok = false;
          if (!ok) break;
          const int s = (int)(it % p.stages);
          if (!mbar_wait(&full[s], (it / p.stages) & 1u, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const unsigned char *st = smem + (size_t)s * p.stage_bytes;
          if (i < p.kb_l) {
            const uint64_t ah = desc_kmajor_sw128(st);
            const uint64_t al = desc_kmajor_sw128(st + p.a_tile_bytes);
            const uint64_t bd = desc_kmajor_sw128(st + 2 * p.a_tile_bytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              umma_f16(d_l, ah + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), p.idesc_l,
                       (i > 0 || kk > 0) ? 1u : 0u);
              umma_f16(d_l, al + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), p.idesc_l, 1u);
            }
          } else {
            const uint64_t ad = desc_kmajor_sw128(st);
            const uint64_t bd = desc_kmajor_sw128(st + p.a_tile_bytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_f16(d_gu, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), p.idesc_gu,
                       (i > p.kb_l || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (i == p.kb_l - 1) umma_commit(lfull);
          if (i == nblk - 1) umma_commit(gfull);
        }
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;           // token row of the tile
    const int h = (warp - 2) >> 2;           // this thread's bank of the unit
    const int64_t t = row;
    const bool valid = t < p.T;
    const int srow = p.k | 1;
    float *stg = stage_rows + (h * kBM + row) * srow;
    uint32_t lt = 0;
    for (int unit = blockIdx.x; unit < p.n_units; unit += gridDim.x, ++lt) {
      const int bank = unit * 2 + h;
      // 1. logits of bank h: mask word, kept channels' sigma (in stg)
      if (!mbar_wait(lfull, lt & 1u, p.err)) break;
      tc_fence_after();
      const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16) + kAccCols + h * 64;
      uint32_t tau;
      int gt;
      bank_threshold(tl, p.k, tau, gt);
      const int need = p.k - gt;
      int eq = 0, cnt = 0;
      uint64_t word = 0ull;
#pragma unroll 1
      for (int g = 0; g < 4; ++g) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tl + g * 16, v);
        tmem_ld_wait();
        uint32_t b = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t key = order_key(__uint_as_float(v[i]));
          const bool take = (key > tau) | ((key == tau) & (eq < need));
          eq += (key == tau);
          b |= (uint32_t)take << i;
          if (take) stg[cnt] = __uint_as_float(v[i]);
          cnt += take;
        }
        word |= (uint64_t)b << (g * 16);
      }
      tc_fence_before();
      mbar_arrive(lempty);
      for (int s1 = 0; s1 < p.k; ++s1) stg[s1] = sigmoid_fast(stg[s1]);
      if (valid && p.mask != nullptr) p.mask[t * p.n_banks + bank] = word;
      // 2. a = sigma(p) g u for bank h: g at columns [h*64, h*64 + 64), u at
      //    [128 + h*64, ...) of the gate/up accumulator
      if (!mbar_wait(gfull, lt & 1u, p.err)) break;
      tc_fence_after();
      const uint32_t tg = tmem_base + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t g[32], u[32];
        tmem_ld_32x32b_x32(tg + h * 64 + c0, g);
        tmem_ld_32x32b_x32(tg + 128 + h * 64 + c0, u);
        tmem_ld_wait();
        if (valid) {
          uint32_t packed[16];
          int rank = __popcll(word & ((1ull << c0) - 1ull));
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float a2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const bool on = (word >> (c0 + i + e)) & 1ull;
              const float sg = on ? stg[rank] : 0.f;
              a2[e] = on ? sg * __uint_as_float(g[i + e]) * __uint_as_float(u[i + e]) : 0.f;
              rank += on;
            }
            packed[i / 2] = pack_bf16x2(a2[0], a2[1]);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(p.act + t * p.ld_out + bank * 64 + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2],
                                packed[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(gempty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

// ------------------------------------------------------------------ host
template <int kEpi>
cudaError_t launch_tc(const CUtensorMap &tA, const CUtensorMap &tB, const CUtensorMap &tB2,
                      TcParams p, int num_sms, cudaStream_t st) {
  using Tr = EpiTraits<kEpi>;
  const uint32_t b_bytes = (uint32_t)p.bn * 128u;  // 64 K-rows of bn elements
  // A tiles hold only the token rows loaded; the MMA still reads kBM rows
  // (kTileA bytes) from each A tile start, which may run past the stage: a
  // tail of kTileA bytes keeps every such read inside the allocation
  const uint32_t a_rows = p.a_rows > 0 ? (uint32_t)p.a_rows : (uint32_t)kBM;
  p.a_tile_bytes = a_rows * (kBK * 2);
  p.stage_bytes = Tr::kNumA * p.a_tile_bytes + b_bytes;
  p.tx_bytes = p.stage_bytes;
  const size_t epi_bytes =
      (kEpi == kEpiTopk) ? (size_t)(Tr::kEpiWarps / 4) * kBM * (p.k | 1) * sizeof(float) : 0;
  // as many stages as fit beside the alignment slack, barriers and staging
  const size_t fixed = 1024 + 256 + epi_bytes + (a_rows < (uint32_t)kBM ? kTileA : 0);
  p.stages = (int)(((size_t)kMaxDynSmem - fixed) / p.stage_bytes);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) return cudaErrorInvalidValue;
  p.idesc = idesc_bf16_f32(kBM, p.bn, Tr::kBMnMajor, Tr::kAMnMajor);
  const size_t smem = fixed + (size_t)p.stages * p.stage_bytes;
  if ((2 * p.stages + 5) * 8 + 4 > 256) return cudaErrorInvalidValue;
  auto kern = k_tc_gemm<kEpi>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int total = p.tiles_m * p.tiles_n * p.ksplit;
  const int grid = total < num_sms ? total : num_sms;
  e = launch_pdl(kern, dim3(grid), dim3(Tr::kThreads), smem, st, tA, tB, tB2, p);
  count_launches(1);
  return e;
}

}  // namespace

bool tc_shape_ok(const FwdShape &s) {
  return s.bf16 && s.bank == 64 && s.d % 256 == 0 && s.d_i % 256 == 0 && s.r % 64 == 0 &&
         s.r <= 512 && s.T > 0 && s.T <= 0x7fffffffLL;
}

TcPlan plan_tc(const FwdShape &s) {
  TcPlan p{};
  p.ksplit = tc_down_splits(s, 148);  // fixed: scratch independent of the device
  p.hsplit = tc_h_splits(s, 148);
  size_t off = 0;
  p.off_h2 = off;
  off = align_up(off + (size_t)s.T * 2 * s.r * 2, 256);
  p.off_sig = off;
  off = align_up(off + (size_t)s.T * s.d_s * 4, 256);
  p.off_act = off;
  off = align_up(off + (size_t)s.T * s.d_i * 2, 256);
  p.off_mask = off;
  off = align_up(off + (size_t)s.T * s.n_banks * 8, 256);
  p.off_part = off;
  if (p.ksplit > 1) off = align_up(off + (size_t)s.T * p.ksplit * s.d * 4, 256);
  p.off_hpart = off;
  if (p.hsplit > 1) off = align_up(off + (size_t)s.T * p.hsplit * s.r * 4, 256);
  p.total = off;
  return p;
}

namespace {
// Token rows per A-operand TMA box: all of them when they fit one tile
// (rounded up to 16), else a whole tile.
int a_box_rows(const FwdShape &s) {
  return s.T < kBM ? (int)((s.T + 15) / 16 * 16) : kBM;
}

TcParams base_params(const FwdShape &s, const DeviceInfo &dev) {
  TcParams p{};
  p.T = s.T;
  p.err = dev.err;
  p.r = s.r;
  p.k = s.k;
  p.n_banks = s.n_banks;
  p.tiles_m = (int)((s.T + kBM - 1) / kBM);
  p.ksplit = 1;
  p.a_rows = a_box_rows(s);
  p.b_once = (p.tiles_m == 1);
  return p;
}
}  // namespace

int tc_down_splits(const FwdShape &s, int num_sms) {
  const int tiles = (int)((s.T + kBM - 1) / kBM) * (s.d / 256);
  const int kblocks = s.d_i / kBK;
  int ks = 1;
  while (tiles * ks * 2 <= num_sms && ks * 2 <= kblocks / 4) ks *= 2;
  return ks;
}

// Widest N tile from `cands` (descending) that still gives every SM a tile.
constexpr bool kWideGateUpOneTile = true;

static int pick_bn(int tiles_m, int n_total, std::initializer_list<int> cands, int num_sms) {
  int last = 0;
  for (int c : cands) {
    if (n_total % c) continue;
    last = c;
    if ((int64_t)tiles_m * (n_total / c) >= num_sms) return c;
  }
  return last;
}

// N tile of the logits GEMMs (the same in the forward and the backward, so
// both see identical logits): one token tile -> two banks per tile, so that
// both epilogue warps of a TMEM lane quadrant have a bank (measured faster
// than one-bank tiles at 8..100 tokens); otherwise enough tiles for the SMs.
int logits_bn(const FwdShape &s, int tiles_m, int num_sms) {
  if (tiles_m == 1 && s.d_i % 128 == 0) return 128;
  return pick_bn(tiles_m, s.d_i, {256, 128, 64}, num_sms);
}

int tc_h_splits(const FwdShape &s, int num_sms) {
  const int tiles = (int)((s.T + kBM - 1) / kBM) * (s.r / 64);
  const int kblocks = s.d / kBK;
  int ks = 1;
  while (tiles * ks * 2 <= num_sms && ks * 2 <= kblocks / 2) ks *= 2;
  return ks;
}

// G1: H = X A^T.  ksplit == 1: written as bf16 hi | lo halves of h2 [T][2r];
// ksplit > 1: fp32 partial sums [T][ksplit][r] into `partial` (the caller
// reduces them and splits hi/lo).
cudaError_t launch_tc_h(const FwdShape &s, const DeviceInfo &dev, const void *x, const void *A,
                        uint16_t *h2, float *partial, int ksplit, cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  const int tiles_m = (int)((s.T + kBM - 1) / kBM);
  const int bn_h = ksplit > 1 ? 64
                              : pick_bn(tiles_m, s.r, {s.r <= 256 ? s.r : s.r / 2, 64}, dev.num_sms);
  CUtensorMap mX, mA;
  if (!make_map(&mX, x, s.d, s.T, 64, a_box_rows(s)) || !make_map(&mA, A, s.d, s.r, 64, bn_h))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.r / bn_h;
  p.k_blocks = s.d / kBK;
  p.ksplit = ksplit;
  p.bn = bn_h;
  if (ksplit > 1) {
    p.out = partial;
    p.ld_out = s.r;
  } else {
    p.out = h2;
    p.ld_out = 2 * s.r;
  }
  return launch_tc<kEpiHSplit>(mX, mA, mA, p, dev.num_sms, st);
}

// G2: logits = (H_hi + H_lo) B^T; raw fp32 (logits != nullptr) or the bank
// top-k fused into the epilogue (mask + sigma(p) of kept channels).
cudaError_t launch_tc_logits(const FwdShape &s, const DeviceInfo &dev, const uint16_t *h2,
                             const void *B, float *logits, uint64_t *mask, float *sig,
                             cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  const int tiles_m = (int)((s.T + kBM - 1) / kBM);
  const int bn = logits_bn(s, tiles_m, dev.num_sms);
  CUtensorMap mH, mB;
  if (!make_map(&mH, h2, 2 * s.r, s.T, 64, a_box_rows(s)) ||
      !make_map(&mB, B, s.r, s.d_i, 64, bn))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.d_i / bn;
  p.k_blocks = s.r / kBK;
  p.bn = bn;
  if (logits != nullptr) {
    p.out = logits;
    p.ld_out = s.d_i;
    return launch_tc<kEpiLogits>(mH, mB, mB, p, dev.num_sms, st);
  }
  p.mask = mask;
  p.sig = sig;
  return launch_tc<kEpiTopk>(mH, mB, mB, p, dev.num_sms, st);
}

// G2 for the backward: logits (float32 [T][d_i]), mask and each bank's
// threshold (midpoint of its k-th and (k+1)-th logits) from the same epilogue.
cudaError_t launch_tc_logits_tau(const FwdShape &s, const DeviceInfo &dev, const uint16_t *h2,
                                 const void *B, float *logits, uint64_t *mask, float *tau,
                                 cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  const int tiles_m = (int)((s.T + kBM - 1) / kBM);
  const int bn = logits_bn(s, tiles_m, dev.num_sms);
  CUtensorMap mH, mB;
  if (!make_map(&mH, h2, 2 * s.r, s.T, 64, a_box_rows(s)) ||
      !make_map(&mB, B, s.r, s.d_i, 64, bn))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.d_i / bn;
  p.k_blocks = s.r / kBK;
  p.bn = bn;
  p.out = logits;
  p.ld_out = s.d_i;
  p.mask = mask;
  p.sig = nullptr;
  p.tau = tau;
  return launch_tc<kEpiTopk>(mH, mB, mB, p, dev.num_sms, st);
}

// G3: [G | U] = X [Wg; Wu]^T -> act = sigma(p) g u on kept channels, 0 elsewhere.
cudaError_t launch_tc_gateup(const FwdShape &s, const DeviceInfo &dev, const void *x,
                             const void *Wg, const void *Wu, const uint64_t *mask,
                             const float *sig, uint16_t *act, cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  const int tiles_m = (int)((s.T + kBM - 1) / kBM);
  // N tile: g and u of 128 channels (two banks) or of 64 channels (one bank).
  // One token tile: every N tile streams the whole x tile again, so the
  // wider tile (half the x traffic per weight byte) wins even with fewer
  // tiles than SMs.
  const int bn = 2 * ((kWideGateUpOneTile && tiles_m == 1 && s.d_i % 128 == 0)
                          ? 128
                          : pick_bn(tiles_m, s.d_i, {128, 64}, dev.num_sms));
  CUtensorMap mX, mG, mU;
  if (!make_map(&mX, x, s.d, s.T, 64, a_box_rows(s)) ||
      !make_map(&mG, Wg, s.d, s.d_i, 64, bn / 2) ||
      !make_map(&mU, Wu, s.d, s.d_i, 64, bn / 2))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.d_i / (bn / 2);
  p.k_blocks = s.d / kBK;
  p.bn = bn;
  p.out = act;
  p.ld_out = s.d_i;
  p.mask = const_cast<uint64_t *>(mask);
  p.sig = const_cast<float *>(sig);
  return launch_tc<kEpiGateUp>(mX, mG, mU, p, dev.num_sms, st);
}

// G2 + G3 at one token tile (T <= 128): logits, bank top-k and a = sigma(p) g u
// in one kernel (k_tc_logits_gateup).  mask (may be null) receives the mask.
bool tc_fused_gateup_ok(const FwdShape &s) {
  return tc_shape_ok(s) && s.T <= kBM && s.d_i % 128 == 0;
}

cudaError_t launch_tc_logits_gateup(const FwdShape &s, const DeviceInfo &dev,
                                    const uint16_t *h2, const void *B, const void *x,
                                    const void *Wg, const void *Wu, uint64_t *mask,
                                    uint16_t *act, cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  if (!tc_fused_gateup_ok(s)) return cudaErrorInvalidValue;
  const int a_rows = a_box_rows(s);
  CUtensorMap mH, mB, mX, mG, mU;
  if (!make_map(&mH, h2, 2 * s.r, s.T, 64, a_rows) || !make_map(&mB, B, s.r, s.d_i, 64, 128) ||
      !make_map(&mX, x, s.d, s.T, 64, a_rows) || !make_map(&mG, Wg, s.d, s.d_i, 64, 128) ||
      !make_map(&mU, Wu, s.d, s.d_i, 64, 128))
    return cudaErrorInvalidValue;
  G23Params p{};
  p.T = s.T;
  p.n_units = s.d_i / 128;
  p.kb_l = s.r / kBK;
  p.kb_gu = s.d / kBK;
  p.r = s.r;
  p.k = s.k;
  p.n_banks = s.n_banks;
  p.ld_out = s.d_i;
  p.act = act;
  p.mask = mask;
  p.err = dev.err;
  p.a_tile_bytes = (uint32_t)a_rows * kBK * 2;
  p.tx_l = 2 * p.a_tile_bytes + 16384;
  p.tx_gu = p.a_tile_bytes + 32768;
  // one stage holds either block kind; the MMA reads 128 rows from each A
  // tile start, which stays inside the stage (a tile <= 16 KB)
  p.stage_bytes = p.a_tile_bytes + 32768;
  p.idesc_l = idesc_bf16_f32(kBM, 128, false);
  p.idesc_gu = idesc_bf16_f32(kBM, 256, false);
  const size_t epi = (size_t)2 * kBM * (s.k | 1) * sizeof(float);
  const size_t fixed = 1024 + 256 + epi;
  p.stages = (int)(((size_t)kMaxDynSmem - fixed) / p.stage_bytes);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2 || (2 * p.stages + 5) * 8 + 4 > 256) return cudaErrorInvalidValue;
  const size_t smem = fixed + (size_t)p.stages * p.stage_bytes;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(k_tc_logits_gateup), smem);
  if (e != cudaSuccess) return e;
  const int grid = p.n_units < dev.num_sms ? p.n_units : dev.num_sms;
  e = launch_pdl(k_tc_logits_gateup, dim3(grid), dim3(kG23Threads), smem, st, mH, mB, mX, mG,
                 mU, p);
  count_launches(1);
  return e;
}

// Dense-4x comparison, first GEMM: [G | U] = X [Wg; Wu]^T -> act =
// silu(g) u kept where |act| is among the k largest of its bank, 0 elsewhere.
cudaError_t launch_tc_dense4x_gateup(const FwdShape &s, const DeviceInfo &dev, const void *x,
                                     const void *Wg, const void *Wu, uint64_t *mask,
                                     uint16_t *act, cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  const int tiles_m = (int)((s.T + kBM - 1) / kBM);
  const int bn = 2 * pick_bn(tiles_m, s.d_i, {128, 64}, dev.num_sms);
  CUtensorMap mX, mG, mU;
  if (!make_map(&mX, x, s.d, s.T, 64, a_box_rows(s)) ||
      !make_map(&mG, Wg, s.d, s.d_i, 64, bn / 2) ||
      !make_map(&mU, Wu, s.d, s.d_i, 64, bn / 2))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.d_i / (bn / 2);
  p.k_blocks = s.d / kBK;
  p.bn = bn;
  p.out = act;
  p.ld_out = s.d_i;
  p.mask = mask;
  return launch_tc<kEpiDense4x>(mX, mG, mU, p, dev.num_sms, st);
}

// G4: Y = act Wd, with Wd [d_i][d] read as an MN-major B operand.  With
// ksplit > 1, y receives fp32 partial sums [T][ksplit][d] instead.
cudaError_t launch_tc_down(const FwdShape &s, const DeviceInfo &dev, const uint16_t *act,
                           const void *Wd, void *y, int ksplit, cudaStream_t st, bool f32_out) {
  if (!encoder()) return cudaErrorNotSupported;
  CUtensorMap mAct, mD;
  if (!make_map(&mAct, act, s.d_i, s.T, 64, a_box_rows(s)) ||
      !make_map(&mD, Wd, s.d, s.d_i, 64, 64))
    return cudaErrorInvalidValue;
  TcParams p = base_params(s, dev);
  p.tiles_n = s.d / 256;
  p.k_blocks = s.d_i / kBK;
  p.ksplit = ksplit;
  p.bn = 256;
  p.out = y;
  p.ld_out = s.d;
  p.f32_out = f32_out;
  return launch_tc<kEpiDown>(mAct, mD, mD, p, dev.num_sms, st);
}

// C[M][ldc] (=, or += when accumulate) A B: bf16 operands, float32
// accumulation and output.  A is [M][K] (lda elements per row), or [K][M]
// when a_mn; B is [N][K] (ldb), or [K][N] when b_mn.  N must be a multiple of
// 64; M and K are arbitrary (the loads zero-fill past them).  The N tile is
// 256 wide from N = 256 up, with the last one cut at N (so N = 448 runs as
// two wide tiles rather than seven 64-wide ones, which keep the MMA pipe far
// from busy).
cudaError_t launch_tc_gemm_f32(const DeviceInfo &dev, int M, int N, int K, const void *A,
                               int lda, bool a_mn, const void *B, int ldb, bool b_mn, float *C,
                               int ldc, bool accumulate, cudaStream_t st) {
  if (!encoder()) return cudaErrorNotSupported;
  if (M <= 0 || K <= 0 || N <= 0 || N % 64 != 0 || (a_mn && !b_mn)) return cudaErrorInvalidValue;
  const int tiles_m = (M + kBM - 1) / kBM;
  const int bn = N >= 256 ? 256 : N;
  CUtensorMap mA, mB;
  const bool okA = a_mn ? make_map(&mA, A, (uint64_t)M, (uint64_t)K, 64, 64, (uint64_t)lda)
                        : make_map(&mA, A, (uint64_t)K, (uint64_t)M, 64, kBM, (uint64_t)lda);
  const bool okB = b_mn ? make_map(&mB, B, (uint64_t)N, (uint64_t)K, 64, 64, (uint64_t)ldb)
                        : make_map(&mB, B, (uint64_t)K, (uint64_t)N, 64, bn, (uint64_t)ldb);
  if (!okA || !okB) return cudaErrorInvalidValue;
  TcParams p{};
  p.T = M;
  p.err = dev.err;
  p.tiles_m = tiles_m;
  p.tiles_n = (N + bn - 1) / bn;
  p.k_blocks = (K + kBK - 1) / kBK;
  p.ksplit = 1;
  p.bn = bn;
  p.out = C;
  p.ld_out = ldc;
  p.accumulate = accumulate;
  p.n_valid = N;
  if (a_mn) return launch_tc<kEpiF32MM>(mA, mB, mB, p, dev.num_sms, st);
  if (b_mn) return launch_tc<kEpiF32KM>(mA, mB, mB, p, dev.num_sms, st);
  return launch_tc<kEpiF32KK>(mA, mB, mB, p, dev.num_sms, st);
}

}  // namespace sfn
