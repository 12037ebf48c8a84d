// Batched decode kernel: BitLinear for 4..64 tokens on layers whose packed
// weights, spread over the SMs, fit in shared memory (2B-class decode).
//
// dashen-tech.com "BitNet.cpp 深度解析", section "3.1 計算コア：整数行列乗算":
// with ternary weights the product is sum_pos - sum_neg.  Here it is taken on
// the int8 tensor-core path of mma.sync.m16n8k32 (s8 weights x s8
// activations, s32 accumulators): weight rows are the 16 MMA rows, tokens the
// 8 MMA columns.  A packed I2_S word holds 16 codes (w + 1), k = 16 j + 4 b + t
// in byte b, bits 2t; its code plane t, (word >> 2t) & 0x03030303, is exactly
// the four bytes of an MMA A-fragment register when the activations sit in
// the kernels' K order (slot 4t + b of each 16-group holds k = 4b + t), and
// (plane | 0x80808080) - 0x01010101, xor 0x80808080, turns each code byte c
// into the signed byte c - 1 = w without borrows between bytes; so the MMA
// gives sum_k x_q w directly and no row sums of x_q are needed.
//
// Work split.  The features are cut into G row groups (as even as integer
// division makes them) and K into S slices, with G * S as close to the SM
// count as it gets: one CTA per SM and layer, so that with programmatic
// dependent launch and two CTAs per SM every SM holds exactly one CTA of the
// running layer and one of the next (a smaller grid lets the scheduler put two
// CTAs of one layer on an SM, which then takes twice as long).  CTA (group,
// slice) keeps the group's packed weights for its slice in shared memory,
// loaded by 16-byte asynchronous copies from every thread before the
// dependency wait (weights never depend on the previous kernel; a slice row is
// only ks/4 bytes, too short for efficient bulk copies, and the shared rows
// are padded).  After the wait the CTA quantises its slice of every token (the
// per-token scale comes from an absmax handed over by the producer of x), the
// warps run the MMAs of their (16-row tile, K part) items, and the partial
// accumulators are staged in shared memory, one copy per K part.  With S > 1 the slices are added into an int32 scratch
// by bulk reductions (cp.reduce.async.bulk .add.s32) and the last CTA of a
// group to arrive -- an arrival counter, no waiting -- dequantises, stores y,
// clears the scratch and the counter again.
//
// Hand-over.  The CTA that stores a group's outputs also takes, per token,
// the largest |y| of its bf16 stores and folds it into amax_out with an
// atomic max, so the next layer of a chain gets its per-token scale without a
// pass over x of its own: that is the absmax its quantiser would compute.
#include "common.cuh"

namespace bitnet {

struct BatchedParams {
  const uint8_t* w;          // packed [N, K/4]
  const float* gamma;
  const uint16_t* x;         // bf16 [M, K]
  uint16_t* y;               // bf16 [M, N]
  float* y_f32;              // optional [M, N]
  int32_t* acc;              // optional [M, N]
  const float* amax_in;      // [M] per-token max |x| (bf16 values)
  unsigned* amax_out;        // optional [M]: atomic max of |y| bits
  float* amax_clear;         // optional [M]: zeroed by CTA 0 after the wait
  int32_t* ws_acc;           // [M, ldw] split-K sums, group g at column g * R
                             // (zero on entry and exit)
  unsigned* ws_cnt;          // [G] arrival counters (zero on entry and exit)
  int N, K, M;
  int G;                     // row groups (rows [g N / G, (g + 1) N / G))
  int RT;                    // 16-row tiles per group (R = 16 RT rows reserved)
  int S;                     // K slices
  int kc;                    // 64-wide K chunks per slice (the last may have fewer)
  int KP;                    // K parts per tile (one warp item each)
  int ldw;                   // row stride of ws_acc (elements)
  uint32_t x_off, w_off;     // shared-memory offsets
  uint32_t xstride, wstride; // bytes per shared token row / weight row
  uint32_t pstride;          // int32 per staged token row
};

constexpr int kBWarps = 8;
constexpr int kBThreads = kBWarps * 32;
constexpr uint32_t kBSmemMax = 112u * 1024u;    // two CTAs per SM
constexpr uint32_t kBHead = 896;                // barrier, token scalars, flag
constexpr int kBMaxGroups = 256;                // ws_acc holds N + 16 * 256 columns

extern __shared__ __align__(128) uint8_t g_bat_smem[];

__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
// c += A (16x32 s8, row-major fragment) * B (32x8 s8, column fragment)
__device__ __forceinline__ void mma_s8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// global[dst .. dst + bytes) += shared[src ..] as int32, by the bulk-copy unit
__device__ __forceinline__ void bulk_reduce_add_s32(int32_t* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.s32 [%0], [%1], %2;" ::"l"(
                   dst),
               "r"(src), "r"(bytes)
               : "memory");
}
// 16-byte global -> shared copy that bypasses L1, with an L2 policy
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst),
               "l"(src), "l"(policy)
               : "memory");
}
// arrive on the mbarrier once all of this thread's earlier cp.async completed
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// NT: groups of 8 tokens (1, 2, 4 or 8); IPW: items (tile, K part) per warp
// (1 or 2); XB: activation loads in flight per thread.
template <int NT, int IPW, int XB>
__global__ void __launch_bounds__(kBThreads, 2)
    batched_kernel(const __grid_constant__ BatchedParams p) {
  uint64_t* bar = reinterpret_cast<uint64_t*>(g_bat_smem);
  float* s_sc = reinterpret_cast<float*>(g_bat_smem + 64);         // [64] token scales
  float* s_td = reinterpret_cast<float*>(g_bat_smem + 320);        // [64] gamma / s
  int* s_flag = reinterpret_cast<int*>(g_bat_smem + 576);
  uint8_t* xq = g_bat_smem + p.x_off;                               // [Mp][xstride]
  uint8_t* wsm = g_bat_smem + p.w_off;                              // [R][wstride]
  int32_t* stage = reinterpret_cast<int32_t*>(g_bat_smem + p.x_off); // [KP][M][pstride], later

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, N = p.N, M = p.M, S = p.S, KP = p.KP;
  const int R = 16 * p.RT;
  const int grp = blockIdx.x / S, sl = blockIdx.x - grp * S;
  const int n0 = (int)((int64_t)grp * N / p.G);
  const int RV = (int)((int64_t)(grp + 1) * N / p.G) - n0;     // rows of this group
  const int c0 = sl * p.kc, c1 = min(c0 + p.kc, K >> 6);
  const int k0 = c0 << 6, ks = (c1 - c0) << 6;
  const uint32_t Rb = (uint32_t)ks >> 2;         // packed bytes per row slice
  const uint32_t wstride = p.wstride, xstride = p.xstride, pstride = p.pstride;

  // ---- weights of the slice: 16-byte chunks dealt to all threads, each
  // thread arriving on the barrier when its own copies have landed
  if (tid == 0) {
    mbar_init(bar, kBThreads);
    fence_mbar_init();
    pdl_launch_dependents();
  }
  __syncthreads();
  {
    const uint64_t pol = policy_evict_first();
    const int cpr = (int)(Rb >> 4);                       // chunks per row
    const uint8_t* wsrc = p.w + (int64_t)n0 * (K >> 2) + (k0 >> 2);
    const uint32_t wdst = smem_u32(wsm);
    for (int i = tid; i < RV * cpr; i += kBThreads) {
      const int r = i / cpr, cc = i - r * cpr;
      cp_async16(wdst + (uint32_t)r * wstride + 16u * cc, wsrc + (int64_t)r * (K >> 2) + 16 * cc,
                 pol);
    }
    cp_async_arrive(bar);
  }

  pdl_wait();

  // ---- this slice of every token: 8-value packs (token m, pack pi) dealt
  // to all threads; the first batch of loads and the token scales (absmax
  // handed over) are in flight together
  const uint32_t x_addr = smem_u32(xq);
  const int npk = ks >> 3, nit = M * npk;
  // (token, pack) of item i: one division per thread up front, then each
  // step of kBThreads items is an addition with a carry
  const int dm = kBThreads / npk, dpi = kBThreads - dm * npk;
  auto advance = [&](int& m, int& pi) {
    pi += dpi;
    m += dm;
    if (pi >= npk) { pi -= npk; ++m; }
  };
  int bm = tid / npk, bpi = tid - bm * npk;    // item of the batch's first step
  uint4 v[XB];
  auto load_batch = [&](int i0) {
    int m = bm, pi = bpi;
#pragma unroll
    for (int b = 0; b < XB; ++b) {
      if (i0 + b * kBThreads < nit)
        v[b] = *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + k0 + 8 * pi);
      advance(m, pi);
    }
  };
  load_batch(tid);
  if (tid < M) {
    const float s = qscale(p.amax_in[tid]);
    s_sc[tid] = s;
    s_td[tid] = __fdiv_rn(*p.gamma, s);
    if (p.amax_clear && blockIdx.x == 0) p.amax_clear[tid] = 0.f;
  }
  __syncthreads();
  for (int i0 = tid; i0 < nit; i0 += XB * kBThreads) {
    if (i0 != tid) load_batch(i0);
    int m = bm, pi = bpi;
#pragma unroll
    for (int b = 0; b < XB; ++b, advance(m, pi)) {
      const int i = i0 + b * kBThreads;
      if (i < nit) {
        const float sc = s_sc[m];
        const uint32_t w[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
        int q[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          q[2 * j] = quant_code_sat(__uint_as_float(w[j] << 16), sc);
          q[2 * j + 1] = quant_code_sat(__uint_as_float(w[j] & 0xffff0000u), sc);
        }
        // k = 16g + 8h + j goes to slot 4 (j % 4) + 2h + j / 4 of group g:
        // per code plane c one 16-bit half (values c and c + 4)
        const uint32_t base =
            x_addr + (uint32_t)m * xstride + (uint32_t)((pi >> 1) * 16 + 2 * (pi & 1));
#pragma unroll
        for (int c = 0; c < 4; ++c)
          sts_u16(base + 4 * c, (uint16_t)__byte_perm((uint32_t)q[c], (uint32_t)q[4 + c], 0x0040));
      }
    }
    bm = m;      // XB steps on: the next batch's first item
    bpi = pi;
  }
  __syncthreads();

  // ---- products: warp w takes items w and w + 8 (tile t, K part kp)
  const int g = lane >> 2, tig = lane & 3;
  const int nks = ks >> 5, nitem = p.RT * KP;
  // independent accumulator sets so that a warp always has 4 or more MMAs
  // in flight (consecutive MMAs on one accumulator wait for each other)
  constexpr int kAcc = NT >= 4 ? 1 : 4 / NT;
  int c[IPW][NT][4];
  bool ok = mbar_wait(bar, 0);
  // ldmatrix rows: lane l addresses row (l & 7) of matrix l >> 3; matrices
  // (group n, first 16 k), (n, last 16 k), (n + 1, first), (n + 1, last)
  const int mj = NT == 1 ? ((lane >> 3) & 1) : (lane >> 3);
  const uint32_t xrow =
      x_addr + (uint32_t)(8 * (mj >> 1) + (lane & 7)) * xstride + 16u * (uint32_t)(mj & 1);
  const int sh = 2 * tig;
#pragma unroll
  for (int ii = 0; ii < IPW; ++ii) {
    const int it = warp + kBWarps * ii;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) c[ii][n][e] = 0;
    if (!ok || it >= nitem) continue;
    const int t = it / KP, kp = it - t * KP;
    const int ka = (kp * nks) / KP, kb = ((kp + 1) * nks) / KP;
    const uint32_t wbase = smem_u32(wsm) + (uint32_t)(16 * t + g) * wstride;
    int ca[kAcc][NT][4];
#pragma unroll
    for (int ac = 0; ac < kAcc; ++ac)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) ca[ac][n][e] = 0;
    auto step = [&](int kst, int (&cc)[NT][4]) {
      const uint2 lo = lds_v2(wbase + 8u * kst);
      const uint2 hi = lds_v2(wbase + 8u * wstride + 8u * kst);
      // code plane -> signed weight bytes (c | 0x80) - 1, xor 0x80 = c - 1
      auto wq = [&](uint32_t word) {
        return (((word >> sh) & 0x03030303u | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
      };
      const uint32_t a[4] = {wq(lo.x), wq(hi.x), wq(lo.y), wq(hi.y)};
      uint32_t b[NT][2];
      if constexpr (NT == 1) {
        ldsm_x2(xrow + 32u * kst, b[0][0], b[0][1]);
      } else {
#pragma unroll
        for (int n = 0; n < NT; n += 2)
          ldsm_x4(xrow + (uint32_t)(8 * n) * xstride + 32u * kst, b[n][0], b[n][1], b[n + 1][0],
                  b[n + 1][1]);
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) mma_s8s8(cc[n], a, b[n][0], b[n][1]);
    };
    int kst = ka;
    for (; kst + kAcc <= kb; kst += kAcc) {
#pragma unroll
      for (int ac = 0; ac < kAcc; ++ac) step(kst + ac, ca[ac]);
    }
#pragma unroll
    for (int ac = 0; ac < kAcc - 1; ++ac)
      if (kst + ac < kb) step(kst + ac, ca[ac]);
#pragma unroll
    for (int ac = 0; ac < kAcc; ++ac)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[ii][n][e] += ca[ac][n][e];
  }
  const bool all_ok = __syncthreads_and(ok) != 0;   // x_q and weights are dead now

  // ---- stage the items: copy kp of token m, row r at (kp M + m) pstride + r
#pragma unroll
  for (int ii = 0; ii < IPW; ++ii) {
    const int it = warp + kBWarps * ii;
    if (it < nitem) {
      const int t = it / KP, kp = it - t * KP;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = 16 * t + g + (e >= 2 ? 8 : 0);
          const int m = 8 * n + 2 * tig + (e & 1);
          if (m < M)
            stage[(kp * M + m) * pstride + r] = c[ii][n][e];
        }
    }
  }
  __syncthreads();

  // ---- dequantise a group's rows from `copies` staged copies: warp w takes
  // tokens w, w + 8, ...
  auto finish = [&](int copies) {
    for (int m = warp; m < M; m += kBWarps) {
      const float td = s_td[m];
      uint32_t hmax = 0;
      for (int r = lane; r < RV; r += 32) {
        int ac = 0;
        for (int q = 0; q < copies; ++q) ac += stage[(q * M + m) * pstride + r];
        const float y32 = __fmul_rn(__int2float_rn(ac), td);
        const uint16_t yb = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
        const int64_t o = (int64_t)m * N + n0 + r;
        p.y[o] = yb;
        if (p.y_f32) p.y_f32[o] = y32;
        if (p.acc) p.acc[o] = ac;
        uint32_t h = yb & 0x7fffu;
        h = h > 0x7f80u ? 0u : h;          // NaN takes no part, as in fmaxf
        hmax = h > hmax ? h : hmax;
      }
      if (p.amax_out) {
        hmax = __reduce_max_sync(0xffffffffu, hmax);
        if (lane == 0) atomicMax(p.amax_out + m, hmax << 16);
      }
    }
  };

  if (S == 1) {
    if (all_ok) finish(KP);
  } else if (all_ok) {
    fence_proxy_async_smem();              // the staged rows, to the bulk-copy unit
    __syncthreads();
    int32_t* wsg = p.ws_acc + grp * R;
    if (warp == 0) {
      for (int i = lane; i < KP * M; i += 32)
        bulk_reduce_add_s32(wsg + (int64_t)(i % M) * p.ldw, smem_u32(stage + i * pstride),
                            (uint32_t)R * 4u);
      bulk_commit();
      bulk_wait0();
      fence_proxy_async_global();
      __threadfence();
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned t = atomicAdd(p.ws_cnt + grp, 1u);
      s_flag[0] = t == (unsigned)(S - 1);
    }
    __syncthreads();
    if (s_flag[0]) {
      // the last slice of the group: read the sums back into the stage (all
      // loads in flight at once, 16 bytes each), clear them, dequantise
      __threadfence();
      const int q4 = R >> 2;                              // 16-byte pieces per token row
      const int nq = M * q4;
      for (int i0 = tid; i0 < nq; i0 += 8 * kBThreads) {
        int4 rv[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int i = i0 + b * kBThreads;
          if (i < nq) {
            const int m = i / q4, cq = i - m * q4;
            rv[b] = __ldcg(reinterpret_cast<const int4*>(wsg + (int64_t)m * p.ldw) + cq);
          }
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int i = i0 + b * kBThreads;
          if (i < nq) {
            const int m = i / q4, cq = i - m * q4;
            __stcg(reinterpret_cast<int4*>(wsg + (int64_t)m * p.ldw) + cq, make_int4(0, 0, 0, 0));
            *reinterpret_cast<int4*>(stage + m * pstride + 4 * cq) = rv[b];
          }
        }
      }
      if (tid == 0) p.ws_cnt[grp] = 0u;
      __syncthreads();
      finish(1);
    }
  }
  if (!all_ok) {
    // a wait gave up (recorded in the status word): let this CTA's copies
    // finish, within the same limit, before its shared memory is released
    if (tid == 0) mbar_wait(bar, 0);
  }
}

// Absmax of each token's bf16 row (a warp per token) into amax[M], and a
// zeroed range of scratch; used ahead of the first batched layer.
__global__ void __launch_bounds__(256) batched_prep_kernel(const uint16_t* x, int M, int K,
                                                           float* amax, uint4* zero,
                                                           int64_t nzero) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (m < M) {
    const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
    float mx = 0.f;
    for (int i = lane; i < (K >> 3); i += 32) {
      const uint4 v = row[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mx = fmaxf(mx, fabsf(__uint_as_float(w[j] << 16)));
        mx = fmaxf(mx, fabsf(__uint_as_float(w[j] & 0xffff0000u)));
      }
    }
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
    if (lane == 0) amax[m] = mx;
  }
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nzero; i += stride)
    zero[i] = make_uint4(0, 0, 0, 0);
}

// Host-side plan.
struct BatchedPlan {
  BatchedParams p;
  int grid;
  uint32_t smem;
  int NT, IPW;
};

static uint32_t bal128(uint64_t v) { return (uint32_t)((v + 127) & ~uint64_t(127)); }

static bool plan_batched(int M, int N, int K, int num_sms, BatchedPlan* out) {
  if (M < 9 || M > 32 || K % 64 != 0 || K > 65536 || N < 1 || num_sms < 1) return false;
  const int NT = M <= 16 ? 2 : 4;
  const int Mp = 8 * NT;
  const int XB = NT <= 2 ? 16 : 8;
  const int chunks = K / 64;
  const int sms = num_sms < kBMaxGroups ? num_sms : kBMaxGroups;
  double best = 1e300;
  bool found = false;
  for (int S = 1; S <= chunks; ++S) {
    const int kc = (chunks + S - 1) / S;
    if ((chunks + kc - 1) / kc != S) continue;        // each slicing once
    int G = sms / S;
    if (G < 1) break;
    if (G > N) G = N;
    const int rvmax = (N + G - 1) / G;
    const int RT = (rvmax + 15) / 16;
    int KP = RT >= kBWarps ? 1 : kBWarps / RT;
    if (KP > 2 * kc) KP = 2 * kc;                     // a 32-wide K step per part
    const int items = RT * KP;
    const int IPW = (items + kBWarps - 1) / kBWarps;
    if (IPW > 2) continue;
    const uint32_t ksm = 64u * (uint32_t)kc;
    const uint32_t xstride = ksm + 16u;               // 8 token rows on distinct banks
    uint32_t wstride = ksm / 4u;                      // stride = 4 (mod 8) words
    if (((ksm / 16u) & 7u) == 0) wstride += 16u;
    const uint32_t R = 16u * (uint32_t)RT;
    const uint32_t pstride = R + 4u;                  // staged writes on distinct banks
    const uint64_t main = bal128((uint64_t)Mp * xstride) + (uint64_t)R * wstride;
    const uint64_t stg = (uint64_t)KP * M * pstride * 4u;
    const uint64_t smem = kBHead + (main > stg ? main : stg);
    if (smem > kBSmemMax) continue;
    // cycle estimate of one CTA: the MMAs (at the SM's int8 mma.sync rate, or
    // a warp's dependent chain), the slice's activations (bytes from L2 and a
    // round trip per batch of loads), the quantisation, staging and stores;
    // split K adds three dependent round trips through L2 (the bulk
    // reduction's completion, the arrival counter, the read-back: about
    // 2.5 us together, measured) and the reduction traffic
    const double steps = 2.0 * kc;
    const double mma_sm = RT * steps * NT * 2.1;
    const double mma_warp = IPW * (steps / KP) * (NT * 2.0 + 10.0);
    const double mma = mma_sm > mma_warp ? mma_sm : mma_warp;
    const double per_thread = (double)M * kc * 8 / kBThreads;
    const double xload = (double)M * ksm / 32.0 + 1400.0 * ((int)(per_thread + XB - 1) / XB);
    const double quant = (double)M * ksm / 32.0;
    const double fin = (double)R * M * KP / 64.0 + (S > 1 ? 5000.0 + (double)R * M / 8.0 : 0.0);
    const double cost = mma + xload + quant + fin;
    if (cost < best) {
      best = cost;
      found = true;
      BatchedParams& q = out->p;
      q = BatchedParams{};
      q.N = N; q.K = K; q.M = M; q.G = G; q.RT = RT; q.S = S; q.kc = kc; q.KP = KP;
      q.x_off = kBHead;
      q.w_off = kBHead + bal128((uint64_t)Mp * xstride);
      q.xstride = xstride; q.wstride = wstride; q.pstride = pstride;
      out->grid = G * S;
      out->smem = (uint32_t)smem;
      out->NT = NT;
      out->IPW = IPW;
    }
  }
  return found;
}

template <int NT, int IPW>
static cudaError_t launch_batched_t(const BatchedPlan& pl, cudaStream_t stream) {
  constexpr int XB = NT <= 2 ? 16 : 8;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attr_once(configured, batched_kernel<NT, IPW, XB>, (int)kBSmemMax,
                                     cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid);
  cfg.blockDim = dim3(kBThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, batched_kernel<NT, IPW, XB>, pl.p);
}

}  // namespace bitnet

using namespace bitnet;

// Whether the batched decode kernel serves this shape: 0 if not, else the
// number of K slices it plans (1: no split-K scratch is touched).
int bitnet_batched_splits(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M > 64 || N > 0x7fffffff || K > 0x7fffffff) return 0;
  BatchedPlan pl;
  return plan_batched((int)M, (int)N, (int)K, num_sms, &pl) ? pl.p.S : 0;
}

bitnet_status bitnet_batched_launch(const uint8_t* w, const float* gamma, int N, int K,
                                    const uint16_t* x, int M, uint16_t* y, float* y_f32,
                                    int32_t* acc, const float* amax_in, unsigned* amax_out,
                                    float* amax_clear, int32_t* ws_acc, int ldw,
                                    unsigned* ws_cnt, int num_sms, cudaStream_t stream) {
  BatchedPlan pl;
  if (!plan_batched(M, N, K, num_sms, &pl)) return BITNET_ERR_UNSUPPORTED;
  if (pl.p.S > 1 && (int64_t)pl.p.G * 16 * pl.p.RT > ldw) return BITNET_ERR_WORKSPACE;
  BatchedParams& p = pl.p;
  p.w = w; p.gamma = gamma; p.x = x; p.y = y; p.y_f32 = y_f32; p.acc = acc;
  p.amax_in = amax_in; p.amax_out = amax_out; p.amax_clear = amax_clear;
  p.ws_acc = ws_acc; p.ws_cnt = ws_cnt; p.ldw = ldw;
  cudaError_t e;
  switch (pl.NT * 4 + pl.IPW) {
    case 2 * 4 + 1: e = launch_batched_t<2, 1>(pl, stream); break;
    case 2 * 4 + 2: e = launch_batched_t<2, 2>(pl, stream); break;
    case 4 * 4 + 1: e = launch_batched_t<4, 1>(pl, stream); break;
    case 4 * 4 + 2: e = launch_batched_t<4, 2>(pl, stream); break;
    default: return BITNET_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_batched_prep_launch(const uint16_t* x, int M, int K, float* amax,
                                         void* zero, size_t zero_bytes, int num_sms,
                                         cudaStream_t stream) {
  const int64_t n16 = (int64_t)(zero_bytes / 16);
  int64_t grid = (M + 7) / 8;
  int64_t zg = (n16 + 255) / 256;
  if (zg > num_sms) zg = num_sms;
  if (zg > grid) grid = zg;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, batched_prep_kernel, x, M, K, amax,
                                     static_cast<uint4*>(zero), n16);
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
