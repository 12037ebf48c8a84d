// Prefill / batched kernel: tcgen05 kind::i8 MMAs with TMEM accumulators.
//
// The matmul with ternary weights is an integer contraction (dashen-tech.com
// "BitNet.cpp 深度解析", section "3.1 計算コア：整数行列乗算"); with many tokens it
// is a dense one, so it runs on the 5th-generation tensor cores:
//
//   D[n, t] = sum_k code[n, k] * x_q[t, k]      (int8 x int8 -> int32, TMEM)
//   acc     = D - sum_k x_q[t, k]               (code = w + 1, so this is sum w*x_q)
//
// Orientation: the MMA's M side (128 rows) is a tile of output features, its
// N side (BN = 32..256 columns) a tile of tokens.  Per K-stage of 128:
//   * warp 0 (one thread) issues TMA loads of the token tile of x_q (already in
//     the kernels' permuted K order, 128B-swizzled) and of the packed 2-bit
//     weight tile (128 rows x 32 bytes);
//   * warps 2..5 unpack the packed tile to int8 codes {0,1,2} straight into
//     the 128B-swizzled K-major layout the MMA descriptor expects: each packed
//     32-bit word becomes the four code planes (w >> 2t) & 0x03030303, which
//     is exactly the permuted order of x_q;
//   * warp 1 (one thread) issues 4 MMAs of K = 32 per stage per weight matrix
//     and commits completion to the stage's barrier;
//   * after the last stage warps 2..5 read the accumulators out of TMEM
//     (32 lanes x 32 columns per load) and apply the epilogue.
// Every wait on a barrier is bounded (see mbar_wait).  TMA loads use no
// cluster multicast.
#include <cuda.h>

#include "common.cuh"

namespace bitnet {

enum GemmMode : int { gLinear = 0, gGlu = 1, gDown = 2 };

struct GemmArgs {
  int M, N, K;
  int ksplit;               // >1: accumulate D into acc_ws with integer atomics
  const float* scale;       // [M] activation scales s
  const int32_t* rowsum;    // [M] sum of x_q
  const float* gamma0;
  const float* gamma1;
  const double* sumsq_h;    // Down: [M] sum of h'^2 over the inner dim (= K)
  const double* sumsq_x;    // Down: [M] sum of x^2 over the block input
  int H;                    // Down: width of the block input
  float eps;
  uint16_t* y;              // Linear/Down [M,N]
  float* y_f32;             // optional [M,N]
  int32_t* acc0;            // optional [M,N]
  int32_t* acc1;            // optional [M,N] (Glu up)
  float* h;                 // Glu [M,N]
  int32_t* acc_ws0;         // split-K accumulators [M,N]
  int32_t* acc_ws1;
  int32_t* tile_cnt;        // split-K, narrow tiles: K-slices done per tile (the last
                            // CTA finishes the tile); null: a finaliser kernel does
  int tma_store;            // 1: bf16 y written through the staged TMA store
};

constexpr int kBM = 128;                 // features per tile (MMA M)
constexpr int kBK = 128;                 // K elements (bytes) per stage
constexpr int kGemmThreads = 448;        // 14 warps: TMA, MMA, 4 unpack, 8 epilogue

template <int BN, int NMAT>
struct GemmCfg {
  // The unpacked weights are the MMA's A operand.  With one matrix and tiles
  // of at most 192 tokens they live in tensor memory (the unpack warps write
  // them with tcgen05.st, the MMA reads them from there), beside two
  // accumulator sets: each stage then moves only the token tile and the
  // packed weights through shared memory.  Otherwise they are staged in
  // shared memory in the 128-byte-swizzled layout.
  static constexpr bool kTS = NMAT == 1 && BN <= 192;
  static constexpr int kB = BN * kBK;                 // x_q tile bytes
  static constexpr int kA = kTS ? 0 : kBM * kBK;      // one unpacked weight tile (shared)
  static constexpr int kP = kBM * (kBK / 4);          // one packed weight tile
  static constexpr int kStage = kB + NMAT * (kA + kP);
  // accumulator sets in TMEM (512 columns): two when they fit
  static constexpr int kAcc = (2 * NMAT * BN <= 512) ? 2 : 1;
  static constexpr int kStages0 = (218 * 1024 - ((NMAT == 1) ? 32 * 128 * 2 : 0)) / kStage;
  static constexpr int kStagesSm = kStages0 > 6 ? 6 : (kStages0 < 2 ? 2 : kStages0);
  // weight stages in TMEM: 32 columns each (128 int8 of K per lane)
  static constexpr int kStagesTm = kTS ? (512 - kAcc * NMAT * BN) / 32 : kStagesSm;
  static constexpr int kStages = kStagesSm < kStagesTm ? kStagesSm : kStagesTm;
  static constexpr int kACol = kAcc * NMAT * BN;      // first weight-stage column (kTS)
  static_assert(!kTS || (kStages >= 2 && kACol + 32 * kStages <= 512), "TMEM columns");
  static constexpr int kCols0 = kTS ? 512 : kAcc * NMAT * BN;
  static constexpr int kTmemCols = kCols0 <= 32 ? 32 : kCols0 <= 64 ? 64 : kCols0 <= 128 ? 128
                                 : kCols0 <= 256 ? 256 : 512;
  static constexpr int kAux = 512;                    // barriers + tmem slot
  static_assert(8 * (4 * kStages + 2 * kAcc) + 4 <= kAux - 16, "barrier area");
  static constexpr int kTok = BN * 12;                // per-token scalars: d0, rowsum, d1-or-f
  // bf16 output staging for the TMA stores: 8 warps x 2 buffers x (8 tokens x 32 features)
  static constexpr int kStaging = (NMAT == 1) ? 32 * kBM * 2 : 0;
  static constexpr size_t kSmem =
      1024 /*align slack*/ + (size_t)kStages * kStage + kAux + kTok + kStaging;
  // instruction descriptor: D s32, A s8, B s8, both K-major, N = BN, M = 128
  static constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fffu);
  d |= (uint64_t)1u << 16;                 // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset
  d |= (uint64_t)1u << 46;                 // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                 // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_mma_i8(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// A (weights) from tensor memory at column a_tmem, B from shared memory.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t dtmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(dtmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive columns of this warp's 32 TMEM lanes, one register each.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 2, 256;" ::: "memory");
}

// Persistent: each CTA walks work units (feature tile, token tile, K split)
// with stride gridDim.x.  The stage ring and its barrier phases run on across
// units; TMEM holds NACC accumulator sets so the epilogue warps drain unit i
// while the MMA warp already accumulates unit i + 1.
// Split-K: the CTA that adds a tile's last K-slice finishes the whole tile
// (features [n0, n0+128) x tokens [t0, t0+bn)) with `nt` threads (`et` =
// 0..nt-1, which meet at epi_sync): the per-token scalars first (IEEE
// division and the RMS factors, once per token), then every output from the
// integer accumulators (added by every K-slice with atomics, read from L2).
template <int MODE>
__device__ __forceinline__ void splitk_finish_tile(const GemmArgs& a, int n0, int t0, int bn,
                                                   int et, int nt, float* tok_d0, int* tok_rs,
                                                   float* tok_x1) {
  for (int c = et; c < bn; c += nt) {
    const int tok = t0 + c;
    float d0 = 0.f, x1 = 0.f;
    int rs = 0;
    if (tok < a.M) {
      const float s = a.scale[tok];
      d0 = __fdiv_rn(*a.gamma0, s);
      if (MODE == gGlu) x1 = __fdiv_rn(*a.gamma1, s);
      rs = a.rowsum[tok];
      if (MODE == gDown) {
        const double eps = (double)a.eps;
        const double r1 = 1.0 / sqrt(a.sumsq_x[tok] / (double)a.H + eps);
        const double r1_3 = r1 * r1 * r1;
        const double r2 = 1.0 / sqrt(r1_3 * r1_3 * (a.sumsq_h[tok] / (double)a.K) + eps);
        x1 = (float)(r1_3 * r2);
      }
    }
    tok_d0[c] = d0;
    tok_rs[c] = rs;
    tok_x1[c] = x1;
  }
  epi_sync();
  for (int idx = et; idx < bn * kBM; idx += nt) {
    const int c = idx / kBM;
    const int tok = t0 + c, n = n0 + idx % kBM;
    if (tok >= a.M || n >= a.N) continue;
    const int64_t o = (int64_t)tok * a.N + n;
    const int ac = __ldcg(a.acc_ws0 + o) - tok_rs[c];
    if (MODE == gGlu) {
      const int au = __ldcg(a.acc_ws1 + o) - tok_rs[c];
      const float g = __fmul_rn(__int2float_rn(ac), tok_d0[c]);
      const float uu = __fmul_rn(__int2float_rn(au), tok_x1[c]);
      const float rg = fmaxf(g, 0.0f);
      a.h[o] = __fmul_rn(__fmul_rn(rg, rg), uu);
      if (a.acc0) a.acc0[o] = ac;
      if (a.acc1) a.acc1[o] = au;
    } else {
      float y32 = __fmul_rn(__int2float_rn(ac), tok_d0[c]);
      if (MODE == gDown) y32 = __fmul_rn(y32, tok_x1[c]);
      a.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
      if (a.y_f32) a.y_f32[o] = y32;
      if (a.acc0) a.acc0[o] = ac;
    }
  }
  epi_sync();   // the scalars are free again
}

template <int MODE, int BN, int NMAT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw0,
                const __grid_constant__ CUtensorMap tw1, const __grid_constant__ CUtensorMap ty,
                const GemmArgs a) {
  using C = GemmCfg<BN, NMAT>;
  constexpr int S = C::kStages;
  constexpr int NACC = C::kAcc;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
  uint8_t* aux = smem + (size_t)S * C::kStage;
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(aux);   // the stage's token tile
  uint64_t* w_full = tma_full + S;                         // the stage's packed weights
  uint64_t* a_full = w_full + S;
  uint64_t* mma_done = a_full + S;
  uint64_t* acc_full = mma_done + S;         // [NACC]
  uint64_t* acc_empty = acc_full + NACC;     // [NACC]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + NACC);
  volatile int* last_flag = reinterpret_cast<volatile int*>(aux + C::kAux - 16);
  float* tok_d0 = reinterpret_cast<float*>(aux + C::kAux);
  int* tok_rs = reinterpret_cast<int*>(tok_d0 + BN);
  float* tok_x1 = reinterpret_cast<float*>(tok_rs + BN);   // Glu: gamma_up / s; Down: r1^3 r2
  float* tok_d1 = tok_x1;
  float* tok_f = tok_x1;
  uint8_t* staging = aux + C::kAux + C::kTok;     // 8 warps x 2 x [8 tokens][32 features] bf16

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles = (a.N + kBM - 1) / kBM;
  const int m_tiles = (a.M + BN - 1) / BN;
  const int units = n_tiles * m_tiles * a.ksplit;
  const int kst = (a.K + kBK - 1) / kBK;

  // unit -> (n_tile, m_tile, kz); feature tiles vary fastest so that the
  // CTAs running at one time share token tiles in L2
  auto decode_unit = [&](int unit, int& nt, int& mt, int& k0, int& nk) {
    nt = unit % n_tiles;
    const int rest = unit / n_tiles;
    mt = rest % m_tiles;
    const int kz = rest / m_tiles;
    k0 = (int)(((int64_t)kz * kst) / a.ksplit);
    nk = (int)(((int64_t)(kz + 1) * kst) / a.ksplit) - k0;
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&w_full[s], 1);
      mbar_init(&a_full[s], 4);
      mbar_init(&mma_done[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    fence_mbar_init();
    prefetch_tmap(&tx);
    prefetch_tmap(&tw0);
    if (NMAT == 2) prefetch_tmap(&tw1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();
      bool waited = false;
      int u = 0;                               // running stage counter
      for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
        int nt, mt, k0, nk;
        decode_unit(unit, nt, mt, k0, nk);
        for (int kk = 0; kk < nk; ++kk, ++u) {
          const int s = u % S;
          if (u >= S && !mbar_wait(&mma_done[s], ((u / S) - 1) & 1)) { u = -1; break; }
          uint8_t* st = smem + (size_t)s * C::kStage;
          const int kx = (k0 + kk) * kBK;
          // weights never depend on the previous kernel: load them first, on
          // their own barrier, so the unpack warps start while the token
          // tile is still arriving
          mbar_arrive_expect_tx(&w_full[s], (uint32_t)(NMAT * C::kP));
          tma_load_2d(st + C::kB + NMAT * C::kA, &tw0, &w_full[s], kx / 4, nt * kBM, pol_w);
          if (NMAT == 2)
            tma_load_2d(st + C::kB + NMAT * C::kA + C::kP, &tw1, &w_full[s], kx / 4, nt * kBM,
                        pol_w);
          if (!waited) { pdl_wait(); waited = true; }
          mbar_arrive_expect_tx(&tma_full[s], (uint32_t)C::kB);
          tma_load_2d(st, &tx, &tma_full[s], kx, mt * BN, pol_x);
        }
        if (u < 0) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int u = 0, i = 0;
      for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x, ++i) {
        int nt, mt, k0, nk;
        decode_unit(unit, nt, mt, k0, nk);
        const int ab = i % NACC;
        if (i >= NACC && !mbar_wait(&acc_empty[ab], ((i / NACC) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(ab * NMAT * BN);
        for (int kk = 0; kk < nk; ++kk, ++u) {
          const int s = u % S;
          const uint32_t ph = (u / S) & 1;
          ok = mbar_wait(&a_full[s], ph) && mbar_wait(&tma_full[s], ph);
          if (!ok) break;
          tc_fence_after();
          uint8_t* st = smem + (size_t)s * C::kStage;
          const uint64_t bdesc = sw128_desc(smem_u32(st));
          if constexpr (C::kTS) {
            // the stage's weights: 32 TMEM columns from kACol + 32 s, 8 per MMA
#pragma unroll
            for (int q = 0; q < kBK / 32; ++q)
              tc_mma_i8_ts(dt, tmem + (uint32_t)(C::kACol + 32 * s + 8 * q), bdesc + 2 * q,
                           C::kIdesc, (kk > 0 || q > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat) {
              const uint64_t adesc = sw128_desc(smem_u32(st + C::kB + mat * C::kA));
#pragma unroll
              for (int q = 0; q < kBK / 32; ++q) {
                // advance 32 bytes of K inside the swizzle atom: +2 in 16-byte units
                tc_mma_i8(dt + mat * BN, adesc + 2 * q, bdesc + 2 * q, C::kIdesc,
                          (kk > 0 || q > 0) ? 1u : 0u);
              }
            }
          }
          tc_commit(&mma_done[s]);
        }
        tc_commit(&acc_full[ab]);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------- unpack warps
    // one weight row each; with the weights in TMEM, warp w writes lanes
    // 32 (w % 4) .. + 31 (the lanes a warp may access), its rows
    const int ut = C::kTS ? 32 * (warp & 3) + lane : tid - 64;
    int u = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
      int nt, mt, k0, nk;
      decode_unit(unit, nt, mt, k0, nk);
      for (int kk = 0; kk < nk; ++kk, ++u) {
        const int s = u % S;
        if (!mbar_wait(&w_full[s], (u / S) & 1)) { ok = false; break; }
        uint8_t* st = smem + (size_t)s * C::kStage;
        if constexpr (C::kTS) {
          // the stage's previous MMA (which read these columns) has completed:
          // its commit came before the producer refilled this stage
          tc_fence_after();
          const uint4* pk = reinterpret_cast<const uint4*>(st + C::kB + ut * (kBK / 4));
          const uint4 p0 = pk[0], p1 = pk[1];
          const uint32_t wv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          uint32_t o[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            o[4 * j] = wv[j] & 0x03030303u;
            o[4 * j + 1] = (wv[j] >> 2) & 0x03030303u;
            o[4 * j + 2] = (wv[j] >> 4) & 0x03030303u;
            o[4 * j + 3] = (wv[j] >> 6) & 0x03030303u;
          }
          tmem_st32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(C::kACol + 32 * s),
                    o);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s]);
        } else {
#pragma unroll
          for (int mat = 0; mat < NMAT; ++mat) {
            const uint4* pk = reinterpret_cast<const uint4*>(st + C::kB + NMAT * C::kA +
                                                             mat * C::kP + ut * (kBK / 4));
            const uint4 p0 = pk[0], p1 = pk[1];
            const uint32_t wv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint8_t* arow = st + C::kB + mat * C::kA + ut * kBK;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t w = wv[j];
              const uint4 o = make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u,
                                         (w >> 4) & 0x03030303u, (w >> 6) & 0x03030303u);
              *reinterpret_cast<uint4*>(arow + ((j ^ (ut & 7)) << 4)) = o;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s]);
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // 8 warps: warp w reads TMEM lanes 32*(w%4).. (its quadrant of features)
    // and one half of the token columns.
    pdl_wait();
    const int ew = warp - 6;                 // 0..7
    const int et = tid - 192;                // 0..255
    const int lb = 32 * (warp & 3);
    const int half = ew >> 2;
    const int cbeg = (BN >= 64) ? half * (BN / 2) : 0;
    const int cend = (BN >= 64) ? cbeg + BN / 2 : (half == 0 ? BN : 0);
    int i = 0;
    for (int unit = blockIdx.x; unit < units; unit += gridDim.x, ++i) {
      int nt, mt, k0, nk;
      decode_unit(unit, nt, mt, k0, nk);
      const int ab = i % NACC;
      if (a.ksplit == 1) {
        epi_sync();                          // previous unit's scalars are consumed
        for (int c = et; c < BN; c += 256) {
          const int tok = mt * BN + c;
          float d0 = 0.f, x1 = 0.f;
          int rs = 0;
          if (tok < a.M) {
            const float s = a.scale[tok];
            d0 = __fdiv_rn(*a.gamma0, s);
            if (MODE == gGlu) x1 = __fdiv_rn(*a.gamma1, s);
            rs = a.rowsum[tok];
            if (MODE == gDown) {
              const double eps = (double)a.eps;
              const double r1 = 1.0 / sqrt(a.sumsq_x[tok] / (double)a.H + eps);
              const double r1_3 = r1 * r1 * r1;
              const double r2 = 1.0 / sqrt(r1_3 * r1_3 * (a.sumsq_h[tok] / (double)a.K) + eps);
              x1 = (float)(r1_3 * r2);
            }
          }
          tok_d0[c] = d0;
          tok_rs[c] = rs;
          tok_x1[c] = x1;
        }
        epi_sync();
      }
      const bool ok = mbar_wait(&acc_full[ab], (i / NACC) & 1);
      tc_fence_after();
      const int n = nt * kBM + lb + lane;
      const uint32_t tbase = tmem + ((uint32_t)lb << 16) + (uint32_t)(ab * NMAT * BN);
      const bool exact_small = a.K <= 33024;  // |acc| < 2^22: integer-pipe conversion
      const bool staged = (NMAT == 1) && a.ksplit == 1 && a.tma_store;
      const bool dbg = (a.y_f32 != nullptr) || (a.acc0 != nullptr);
      for (int c0 = cbeg; c0 < cend && ok; c0 += 32) {
        uint32_t v0[32], v1[32];
        tmem_ld32(tbase + c0, v0);
        if (NMAT == 2) tmem_ld32(tbase + BN + c0, v1);
        if (staged) {
          // each warp stages 8 tokens x its 32 features (512 B) per TMA store;
          // two buffers per warp, reused once the store two steps back has
          // finished reading
          const uint32_t wbuf = smem_u32(staging) + (uint32_t)(ew * 1024);
#pragma unroll
          for (int sub = 0; sub < 4; ++sub) {
            const uint32_t buf = wbuf + (uint32_t)(sub & 1) * 512u;
            const int cs = c0 + 8 * sub;
            const uint4 dA = lds_v4(smem_u32(tok_d0 + cs)), dB = lds_v4(smem_u32(tok_d0 + cs + 4));
            const uint4 rA = lds_v4(smem_u32(tok_rs + cs)), rB = lds_v4(smem_u32(tok_rs + cs + 4));
            const float d8[8] = {__uint_as_float(dA.x), __uint_as_float(dA.y), __uint_as_float(dA.z),
                                 __uint_as_float(dA.w), __uint_as_float(dB.x), __uint_as_float(dB.y),
                                 __uint_as_float(dB.z), __uint_as_float(dB.w)};
            const int r8[8] = {(int)rA.x, (int)rA.y, (int)rA.z, (int)rA.w,
                               (int)rB.x, (int)rB.y, (int)rB.z, (int)rB.w};
            float f8[8];
            if (MODE == gDown) {
              const uint4 fA = lds_v4(smem_u32(tok_f + cs)), fB = lds_v4(smem_u32(tok_f + cs + 4));
              f8[0] = __uint_as_float(fA.x); f8[1] = __uint_as_float(fA.y);
              f8[2] = __uint_as_float(fA.z); f8[3] = __uint_as_float(fA.w);
              f8[4] = __uint_as_float(fB.x); f8[5] = __uint_as_float(fB.y);
              f8[6] = __uint_as_float(fB.z); f8[7] = __uint_as_float(fB.w);
            }
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
              const int q = 8 * sub + qq;
              const int ac = (int)v0[q] - r8[qq];
              const float af = exact_small ? small_int_to_float(ac) : __int2float_rn(ac);
              float y32 = __fmul_rn(af, d8[qq]);
              if (MODE == gDown) y32 = __fmul_rn(y32, f8[qq]);
              asm volatile("st.shared.u16 [%0], %1;" ::"r"(buf + (uint32_t)(qq * 64 + lane * 2)),
                           "h"((unsigned short)f32_to_bf16_rne_bits(y32)));
              if (dbg) {
                const int tok = mt * BN + cs + qq;
                if (tok < a.M && n < a.N) {
                  const int64_t o = (int64_t)tok * a.N + n;
                  if (a.y_f32) a.y_f32[o] = y32;
                  if (a.acc0) a.acc0[o] = ac;
                }
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&ty, staging + (buf - smem_u32(staging)), nt * kBM + lb, mt * BN + cs);
              bulk_commit();
            }
          }
          continue;
        }
        if (n < a.N) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int c = c0 + q;
            const int tok = mt * BN + c;
            if (tok >= a.M) continue;
            const int64_t o = (int64_t)tok * a.N + n;
            if (a.ksplit > 1) {
              atomicAdd(&a.acc_ws0[o], (int)v0[q]);
              if (NMAT == 2) atomicAdd(&a.acc_ws1[o], (int)v1[q]);
              continue;
            }
            const int ac = (int)v0[q] - tok_rs[c];
            const float af = exact_small ? small_int_to_float(ac) : __int2float_rn(ac);
            if (MODE == gGlu) {
              const int au = (int)v1[q] - tok_rs[c];
              const float auf = exact_small ? small_int_to_float(au) : __int2float_rn(au);
              const float g = __fmul_rn(af, tok_d0[c]);
              const float uu = __fmul_rn(auf, tok_d1[c]);
              const float rg = fmaxf(g, 0.0f);
              a.h[o] = __fmul_rn(__fmul_rn(rg, rg), uu);
              if (a.acc0) a.acc0[o] = ac;
              if (a.acc1) a.acc1[o] = au;
            } else {
              float y32 = __fmul_rn(af, tok_d0[c]);
              if (MODE == gDown) y32 = __fmul_rn(y32, tok_f[c]);
              a.y[o] = (uint16_t)f32_to_bf16_rne_bits(y32);
              if (a.y_f32) a.y_f32[o] = y32;
              if (a.acc0) a.acc0[o] = ac;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      if (a.ksplit > 1 && a.tile_cnt) {
        // the CTA that adds a tile's last K-slice finishes the tile (a
        // counter per tile, cleared with the accumulators before the launch)
        epi_sync();                          // every partial of this unit is added
        if (et == 0) {
          __threadfence();
          *last_flag = atomicAdd(&a.tile_cnt[mt * n_tiles + nt], 1) == a.ksplit - 1;
        }
        epi_sync();
        if (*last_flag) {
          __threadfence();
          splitk_finish_tile<MODE>(a, nt * kBM, mt * BN, BN, et, 256, tok_d0, tok_rs, tok_x1);
        }
      }
    }
  }
  if (warp >= 6 && lane == 0) bulk_wait0();  // this warp's TMA stores have landed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA has completed once the last accumulator set was committed
    // and drained (the epilogue waited on it); wait on the final commit too
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::kTmemCols)
                 : "memory");
  }
}

// Split-K finalisation: integer accumulators -> the mode's epilogue.
template <int MODE>
__global__ void __launch_bounds__(256) splitk_finalize_kernel(const GemmArgs a) {
  pdl_wait();
  const int64_t total = (int64_t)a.M * a.N;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int tok = (int)(o / a.N);
    const float s = a.scale[tok];
    const int rs = a.rowsum[tok];
    const int ac = a.acc_ws0[o] - rs;
    if (MODE == gGlu) {
      const int au = a.acc_ws1[o] - rs;
      const float g = __fmul_rn(__int2float_rn(ac), __fdiv_rn(*a.gamma0, s));
      const float uu = __fmul_rn(__int2float_rn(au), __fdiv_rn(*a.gamma1, s));
      const float rg = fmaxf(g, 0.0f);
      a.h[o] = __fmul_rn(__fmul_rn(rg, rg), uu);
      if (a.acc0) a.acc0[o] = ac;
      if (a.acc1) a.acc1[o] = au;
    } else {
      float y32 = __fmul_rn(__int2float_rn(ac), __fdiv_rn(*a.gamma0, s));
      if (MODE == gDown) {
        const double eps = (double)a.eps;
        const double r1 = 1.0 / sqrt(a.sumsq_x[tok] / (double)a.H + eps);
        const double r1_3 = r1 * r1 * r1;
        const double r2 = 1.0 / sqrt(r1_3 * r1_3 * (a.sumsq_h[tok] / (double)a.K) + eps);
        y32 = __fmul_rn(y32, (float)(r1_3 * r2));
      }
      a.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
      if (a.y_f32) a.y_f32[o] = y32;
      if (a.acc0) a.acc0[o] = ac;
    }
  }
  pdl_launch_dependents();
}

}  // namespace bitnet

// ------------------------------------------------------------------ host
using namespace bitnet;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D tensor map: inner extent `inner` elements, `rows` rows, row stride
// `stride` bytes, box `box_inner` x `box_rows` elements.
static bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                        uint64_t inner, uint64_t rows, uint64_t stride, uint32_t box_inner,
                        uint32_t box_rows, bool sw128) {
  (void)esize;
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE, int BN, int NMAT>
static cudaError_t launch_gemm_t(const CUtensorMap& tx, const CUtensorMap& tw0,
                                 const CUtensorMap& tw1, const CUtensorMap& ty, const GemmArgs& a,
                                 dim3 grid, cudaStream_t stream) {
  using C = GemmCfg<BN, NMAT>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attr_once(configured, gemm_kernel<MODE, BN, NMAT>, (int)C::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<MODE, BN, NMAT>, tx, tw0, tw1, ty, a);
}

// Token-tile width: small M takes the smallest tile that covers it; large M
// picks among 256, 192 and 128 the width whose tile count fills the last
// wave of the persistent grid best (ties to the wider tile).
int bitnet_gemm_pick_bn(int M, int N, int num_sms) {
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  const int cand[3] = {256, 192, 128};
  int best = 256;
  double best_score = -1.0;
  for (int i = 0; i < 3; ++i) {
    const int bn = cand[i];
    const long long mt = (M + bn - 1) / bn;
    const long long units = (long long)((N + kBM - 1) / kBM) * mt;
    const double waves = (double)units / num_sms;
    const double fill = waves / (double)((units + num_sms - 1) / num_sms);
    const double pad = (double)M / (double)(mt * bn);
    // narrower tiles move more shared-memory bytes per MMA: only worth it
    // when they fill the last wave much better
    const double score = fill * pad * (bn == 256 ? 1.0 : (bn == 192 ? 0.85 : 0.75));
    if (score > best_score + 1e-9) { best_score = score; best = bn; }
  }
  return best;
}

// Launch the tensor-core kernel.  With ksplit > 1 the caller has cleared
// acc_ws0 (and acc_ws1) and, for 32-token tiles, tile_cnt: the last CTA of a
// tile finishes it in the kernel; wider tiles (more outputs than one CTA
// should finish at the end) go through the finaliser kernel.
// xq: [M, K] int8 in the permuted K order; w0/w1: packed [N, K/4].
bitnet_status bitnet_gemm_launch(int mode, const int8_t* xq, const uint8_t* w0,
                                 const uint8_t* w1, GemmArgs a, int bn, int num_sms,
                                 cudaStream_t stream) {
  CUtensorMap tx, tw0, tw1;
  const int nmat = mode == gGlu ? 2 : 1;
  if (!make_map_2d(&tx, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K, (uint64_t)a.M,
                   (uint64_t)a.K, kBK, (uint32_t)bn, true))
    return BITNET_ERR_CUDA;
  if (!make_map_2d(&tw0, w0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K / 4, (uint64_t)a.N,
                   (uint64_t)a.K / 4, kBK / 4, kBM, false))
    return BITNET_ERR_CUDA;
  if (nmat == 2) {
    if (!make_map_2d(&tw1, w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.K / 4, (uint64_t)a.N,
                     (uint64_t)a.K / 4, kBK / 4, kBM, false))
      return BITNET_ERR_CUDA;
  } else {
    tw1 = tw0;
  }
  // bf16 output through TMA stores when the row pitch allows (N*2 % 16 == 0)
  CUtensorMap ty = tw0;
  a.tma_store = 0;
  if (nmat == 1 && a.ksplit == 1 && a.N % 8 == 0 &&
      (reinterpret_cast<uintptr_t>(a.y) & 15u) == 0) {
    if (make_map_2d(&ty, a.y, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)a.N, (uint64_t)a.M,
                    (uint64_t)a.N * 2, 32, 8, false))
      a.tma_store = 1;
  }
  if (bn > 32) a.tile_cnt = nullptr;
  const int64_t units = (int64_t)((a.N + kBM - 1) / kBM) * ((a.M + bn - 1) / bn) * a.ksplit;
  dim3 grid((unsigned)(units < num_sms ? units : num_sms));
  cudaError_t e = cudaErrorInvalidValue;
#define BITNET_GEMM_BN(MODE_, NMAT_)                                              \
  switch (bn) {                                                                   \
    case 32: e = launch_gemm_t<MODE_, 32, NMAT_>(tx, tw0, tw1, ty, a, grid, stream); break;   \
    case 64: e = launch_gemm_t<MODE_, 64, NMAT_>(tx, tw0, tw1, ty, a, grid, stream); break;   \
    case 128: e = launch_gemm_t<MODE_, 128, NMAT_>(tx, tw0, tw1, ty, a, grid, stream); break; \
    case 192: e = launch_gemm_t<MODE_, 192, NMAT_>(tx, tw0, tw1, ty, a, grid, stream); break; \
    default: e = launch_gemm_t<MODE_, 256, NMAT_>(tx, tw0, tw1, ty, a, grid, stream); break;  \
  }
  if (mode == gLinear) { BITNET_GEMM_BN(gLinear, 1) }
  else if (mode == gGlu) { BITNET_GEMM_BN(gGlu, 2) }
  else { BITNET_GEMM_BN(gDown, 1) }
#undef BITNET_GEMM_BN
  if (e != cudaSuccess) return BITNET_ERR_CUDA;
  if (a.ksplit > 1 && !a.tile_cnt) {
    cudaLaunchConfig_t cfg = {};
    const int64_t total = (int64_t)a.M * a.N;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (mode == gLinear) e = cudaLaunchKernelEx(&cfg, splitk_finalize_kernel<gLinear>, a);
    else if (mode == gGlu) e = cudaLaunchKernelEx(&cfg, splitk_finalize_kernel<gGlu>, a);
    else e = cudaLaunchKernelEx(&cfg, splitk_finalize_kernel<gDown>, a);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
  }
  return BITNET_OK;
}
