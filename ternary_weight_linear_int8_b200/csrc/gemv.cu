// Decode kernel (M <= 8 tokens): streams packed ternary weights from HBM
// through a shared-memory ring filled by bulk async copies, with the per-token
// activation quantisation fused into its prologue.
//
// dashen-tech.com "BitNet.cpp 深度解析", section "3.1 計算コア：整数行列乗算":
// the product with ternary weights is sum_pos - sum_neg.  Here it is taken in
// the offset form sum_k x_q * code - sum_k x_q (code = w + 1 in {0,1,2}), so a
// packed 32-bit word of 16 codes needs only four AND masks and four dp4a:
// plane t = word & (0x03030303 << 2t) holds, byte b, the code of k = 4b + t
// times 4^t, and the activations sit in shared memory in the matching order.
//
// Layout of work: one CTA per SM owns a contiguous range of output rows.
// The last warp is the producer: bulk copies of whole rows into a ring of
// stages, several stages ahead.  The consumer warps take (block of RB rows,
// K-slice) items, dealt round robin and continuing from stage to stage; lane
// l reads words l, l+32, ... of each row, a butterfly reduction across the
// warp gives each row's partial sum, and either the warp finishes the row
// itself (one slice per block) or shared-memory integer atomics and a
// per-block counter let the warp that adds the last slice finish it.  No
// stage waits for all warps.
//
// Programmatic dependent launch: the producer starts streaming weights
// before griddepcontrol.wait, the consumers wait before reading activations,
// so a kernel's weight stream overlaps the end of the kernel before it.
#include "common.cuh"

namespace bitnet {

enum GemvMode : int { kLinear = 0, kGlu = 1, kDown = 2 };

// Arguments of one decode launch (one BitLinear, or one FFN step).
struct DecodeOp {
  const uint8_t* w0;      // packed [N, K/4]   (Glu: gate)
  const float* gamma0;
  const uint8_t* w1;      // Glu: up
  const float* gamma1;
  const void* x;          // Linear/Glu: bf16 [M,K]; Down: fp32 h' [M,K]
  const float* gain;      // optional [K] (RMSNorm weight)
  const uint16_t* xnorm;  // Down: block input x [M,H] (for r1)
  uint16_t* y;            // Linear/Down [M,N]
  float* y_f32;           // optional [M,N]
  int32_t* acc0;          // optional [M,N]
  int32_t* acc1;          // optional [M,N] (Glu up)
  float* h;               // Glu output h' [M,N]
  int8_t* xq_dbg;         // optional natural-layout x_q [M,K], written by CTA 0
  int N, K, H;
  float eps;
  int mode;
  int rb;                 // rows per work block (4, or 8 for one long-row matrix)
  int rows_per_stage;     // multiple of rb
  int wk;                 // K-slices per row block (a power of two)
};

// Kernel parameters: the op and the shared-memory plan.
struct DecodeParams {
  DecodeOp op;
  int M, stages;
  uint32_t stage_bytes;   // bytes per ring stage (a multiple of 16)
  uint32_t xbytes;        // bytes of the activation area (a multiple of 128)
  uint32_t acc_words;     // integer accumulators per ring stage
  uint32_t cnt_words;     // per-block completion counters per ring stage
};

// 15 consumer warps + 1 producer: 4 warps per scheduler, so up to 128
// registers per thread at one CTA per SM.
constexpr int kConsumerWarps = 15;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxTok = 8;
constexpr uint32_t kCopyChunk = 4096;   // bytes per bulk copy (a multiple of 16)

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Warp-level integer MMA, D = A(16x32, u8, row) * B(32x8, s8, col) + C.
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t u4_at(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Halving step of the butterfly: n values -> n/2, exchanging with lane ^ off.
template <int N>
__device__ __forceinline__ void halve(const int (&v)[N], int (&o)[N / 2], int off, int lane) {
  const bool hi = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const int keep = hi ? v[i + N / 2] : v[i];
    const int send = hi ? v[i] : v[i + N / 2];
    o[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

// 16 consecutive activations (one group) as floats: two 16-byte loads of
// bf16 bits, or four of fp32.
template <bool kF32>
__device__ __forceinline__ void load_group16(const void* x, int64_t idx, float (&v)[16]) {
  if (kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + idx);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = p[i];
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + idx);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 t = p[i];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
        v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
  }
}

__device__ __forceinline__ void load_gain16(const float* g, int64_t idx, float (&v)[16]) {
  const float4* p = reinterpret_cast<const float4*>(g + idx);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 t = p[i];
    v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
  }
}

// Dynamic shared memory of the decode kernel: [0,128) full/empty mbarriers
// (up to 8 stages each); [128,512) per-token scalars; [512,4096) warp
// partials; then the
// permuted activations (xbytes), per ring stage the integer accumulators
// (acc_words) and block counters (cnt_words), and the ring (stages x
// stage_bytes).  Fixed areas are addressed from the array itself, so they
// cost no registers.
extern __shared__ __align__(128) uint8_t g_decode_smem[];

struct DecodeSmem {   // the variable part of the layout (from the plan)
  int S;
  uint32_t stage_bytes, xbytes, acc_words, cnt_words;
  __device__ __forceinline__ uint64_t* full() const {
    return reinterpret_cast<uint64_t*>(g_decode_smem);
  }
  __device__ __forceinline__ uint64_t* empty() const { return full() + 8; }
  __device__ __forceinline__ float* tok_d0() const {
    return reinterpret_cast<float*>(g_decode_smem + 128 + 4 * kMaxTok);
  }
  __device__ __forceinline__ float* tok_d1() const { return tok_d0() + kMaxTok; }
  __device__ __forceinline__ float* tok_f() const { return tok_d1() + kMaxTok; }
  __device__ __forceinline__ float* red_f() const {   // [warps][8 tok]
    return reinterpret_cast<float*>(g_decode_smem + 512);
  }
  __device__ __forceinline__ int* red_i() const {     // [warps][8]
    return reinterpret_cast<int*>(g_decode_smem + 1024);
  }
  __device__ __forceinline__ double* red_d() const {  // [warps][8][2]
    return reinterpret_cast<double*>(g_decode_smem + 2048);
  }
  __device__ __forceinline__ uint8_t* xperm() const { return g_decode_smem + 4096; }
  __device__ __forceinline__ int* acc_s() const {
    return reinterpret_cast<int*>(g_decode_smem + 4096 + xbytes);
  }
  __device__ __forceinline__ int* cnt_s() const {
    return acc_s() + ((S * acc_words + 31) / 32) * 32;
  }
  __device__ __forceinline__ uint8_t* ring() const {
    return g_decode_smem + 4096 + xbytes + ((S * acc_words + 31) / 32) * 128 +
           ((S * cnt_words + 31) / 32) * 128;
  }
};

__device__ __forceinline__ void op_rows(const DecodeOp& o, int& n0, int& n1) {
  n0 = (int)(((int64_t)blockIdx.x * o.N) / gridDim.x);
  n1 = (int)(((int64_t)(blockIdx.x + 1) * o.N) / gridDim.x);
}

// Producer (one thread): bulk copies of this CTA's rows into the ring.
__device__ __forceinline__ void produce(const DecodeOp& o, const DecodeSmem& sm) {
  const uint64_t pol = policy_evict_first();
  const int S = sm.S;
  const bool two = o.mode == kGlu;
  const int Kb = o.K >> 2;
  int n0, n1;
  op_rows(o, n0, n1);
  const int RS = o.rows_per_stage;
  const int nchunks = (n1 - n0 + RS - 1) / RS;
  for (int c = 0; c < nchunks; ++c) {
    const int s = c % S;
    if (c >= S && !mbar_wait(&sm.empty()[s], ((c / S) - 1) & 1)) return;
    const int r0 = n0 + c * RS;
    const int nr = min(RS, n1 - r0);
    const uint32_t bytes = (uint32_t)nr * Kb;
    mbar_arrive_expect_tx(&sm.full()[s], two ? 2 * bytes : bytes);
    uint8_t* dst = sm.ring() + (size_t)s * sm.stage_bytes;
    // several 4 KB copies per stage keep more requests in flight than one
    // large copy
    for (uint32_t off = 0; off < bytes; off += kCopyChunk) {
      const uint32_t nb = bytes - off < kCopyChunk ? bytes - off : kCopyChunk;
      bulk_g2s(dst + off, o.w0 + (int64_t)r0 * Kb + off, nb, &sm.full()[s], pol);
      if (two)
        bulk_g2s(dst + (size_t)RS * Kb + off, o.w1 + (int64_t)r0 * Kb + off, nb, &sm.full()[s],
                 pol);
    }
  }
}

// Consumers: prologue (quantise the input into the permuted layout) and
// main loop over this CTA's stages.  A failed wait (ring_ok false) skips the
// arithmetic and the stores but keeps the ring moving.
template <int MODE, int MT, int MM, int RB>
__device__ __forceinline__ void run_op(const DecodeOp& a, const int M, const DecodeSmem& sm,
                                       bool& ring_ok) {
  // MM: token count rounded up to 1, 2, 4 or 8 (loops over tokens unroll to
  // MM, keeping the code small for single-token decode)
  constexpr int NMAT = (MODE == kGlu) ? 2 : 1;
  // RB: rows per work block (per matrix); NR values per lane per block
  constexpr int NR = RB * NMAT;
  // RB 16: tensor-core items (16-row tiles, all tokens in one MMA column set)
  constexpr bool kMma = RB == 16;
  static_assert(kMma || NR == 4 || NR == 8, "4 or 8 values per block");
  constexpr bool kF32Src = (MODE == kDown);
  constexpr int NT = kConsumerWarps * 32;
  float* tok_d0 = sm.tok_d0();
  float* tok_d1 = sm.tok_d1();
  float* tok_f = sm.tok_f();
  float* red_f = sm.red_f();
  int* red_i = sm.red_i();
  double* red_d = sm.red_d();
  uint8_t* xperm = sm.xperm();
  const int K = a.K, N = a.N;
  const int Mpad = ((M + MT - 1) / MT) * MT;
  const int RS = a.rows_per_stage, S = sm.S, WK = a.wk;   // WK is a power of two
  const int wk_log2 = __ffs(WK) - 1;
  const int acc_words = (int)sm.acc_words;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Kb = K >> 2;                   // bytes per packed row
  const int Kw = K >> 4;                   // 32-bit words per packed row
  int n0, n1;
  op_rows(a, n0, n1);
  const int nchunks = (n1 - n0 + RS - 1) / RS;
  int gs = 0;            // ring stage of the current chunk
  uint32_t gph = 0;      // its phase parity

  // -------------------------------------------------------------- prologue
  // gamma loads go out with the activation loads (their latencies overlap)
  float gam0 = 0.f, gam1 = 0.f;
  if (tid < M) {
    gam0 = *a.gamma0;
    if (MODE == kGlu) gam1 = *a.gamma1;
  }
  for (int i = M * K + tid * 16; i < Mpad * K; i += NT * 16)
    *reinterpret_cast<uint4*>(xperm + i) = make_uint4(0, 0, 0, 0);

  // pass 1: per-token absmax of src*gain (and, for Down, sums of squares).
  // With one or two tokens and at most KEEPG groups of 16 per thread the
  // values stay in registers for pass 2 instead of being loaded again.
  auto load_x = [&](int m, int g, float (&v)[16]) {
    load_group16<kF32Src>(a.x, (int64_t)m * K + g * 16, v);
  };
  constexpr int KEEPG = (MM == 1) ? 2 : 1;
  const bool keep = (MM <= 2) && Kw <= KEEPG * NT;
  float vk[KEEPG][MM][16];
  float am[MM];
  double ss[MM], sx[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) { am[m] = 0.f; ss[m] = 0.0; sx[m] = 0.0; }
  if (keep) {
#pragma unroll
    for (int gi = 0; gi < KEEPG; ++gi) {
      const int g = tid + gi * NT;
      if (g < Kw) {
        float gn[16];
        if (a.gain) load_gain16(a.gain, (int64_t)g * 16, gn);
#pragma unroll
        for (int m = 0; m < MM; ++m) {
          if (m < M) {
            load_x(m, g, vk[gi][m]);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float v = vk[gi][m][i];
              const float vg = a.gain ? __fmul_rn(v, gn[i]) : v;
              am[m] = fmaxf(am[m], fabsf(vg));
              if (MODE == kDown) ss[m] += (double)v * (double)v;
            }
          }
        }
      }
    }
  } else {
#pragma unroll 2
    for (int g = tid; g < Kw; g += NT) {
      float gn[16];
      if (a.gain) load_gain16(a.gain, (int64_t)g * 16, gn);
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        if (m < M) {
          float v[16];
          load_x(m, g, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float vg = a.gain ? __fmul_rn(v[i], gn[i]) : v[i];
            am[m] = fmaxf(am[m], fabsf(vg));
            if (MODE == kDown) ss[m] += (double)v[i] * (double)v[i];
          }
        }
      }
    }
  }
  if (MODE == kDown) {
#pragma unroll 2
    for (int g = tid; g < (a.H >> 4); g += NT) {
#pragma unroll
      for (int m = 0; m < MM; ++m)
        if (m < M) {
          float v[16];
          load_group16<false>(a.xnorm, (int64_t)m * a.H + g * 16, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) sx[m] += (double)v[i] * (double)v[i];
        }
    }
  }
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    if (m < M) {
      const float w = warp_max(am[m]);
      if (lane == 0) red_f[warp * kMaxTok + m] = w;
      if (MODE == kDown) {
        const double d1 = warp_sum_d(ss[m]);
        const double d2 = warp_sum_d(sx[m]);
        if (lane == 0) {
          red_d[(warp * kMaxTok + m) * 2 + 0] = d1;
          red_d[(warp * kMaxTok + m) * 2 + 1] = d2;
        }
      }
    }
  }
  consumer_sync();
  // every thread derives the token scales from the 8 warp maxima itself
  // (same values, same order -> identical in every thread)
  float sc[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    float amax = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) amax = fmaxf(amax, red_f[w * kMaxTok + m]);
    sc[m] = qscale(amax);
  }
  if (tid < M) {
    const int m = tid;
    float s = sc[0];
#pragma unroll
    for (int mm = 1; mm < MM; ++mm) if (mm == m) s = sc[mm];
    tok_d0[m] = __fdiv_rn(gam0, s);
    if (MODE == kGlu) tok_d1[m] = __fdiv_rn(gam1, s);
    if (MODE == kDown) {
      double s1 = 0.0, s2 = 0.0;
      for (int w = 0; w < kConsumerWarps; ++w) {
        s1 += red_d[(w * kMaxTok + m) * 2 + 0];
        s2 += red_d[(w * kMaxTok + m) * 2 + 1];
      }
      const double eps = (double)a.eps;
      const double r1 = 1.0 / sqrt(s2 / (double)a.H + eps);
      const double r1_3 = r1 * r1 * r1;
      const double r2 = 1.0 / sqrt(r1_3 * r1_3 * (s1 / (double)K) + eps);
      tok_f[m] = (float)(r1_3 * r2);
    }
  }
  // pass 2: quantise into the permuted layout, one group of 16 per step
  int rs[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) rs[m] = 0;
  auto quant_group = [&](int g, int m, const float (&v)[16], const float (&gn)[16]) {
    const float s = sc[m];
    int q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float vg = a.gain ? __fmul_rn(v[i], gn[i]) : v[i];
      q[i] = quant_code(vg, s);
      rs[m] += q[i];
    }
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t)
      w[t] = (uint32_t)(q[t] & 0xff) | ((uint32_t)(q[4 + t] & 0xff) << 8) |
             ((uint32_t)(q[8 + t] & 0xff) << 16) | ((uint32_t)(q[12 + t] & 0xff) << 24);
    *reinterpret_cast<uint4*>(xperm + (int64_t)m * K + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    if (a.xq_dbg && blockIdx.x == 0) {
#pragma unroll
      for (int i = 0; i < 16; ++i) a.xq_dbg[(int64_t)m * K + g * 16 + i] = (int8_t)q[i];
    }
  };
  if (keep) {
#pragma unroll
    for (int gi = 0; gi < KEEPG; ++gi) {
      const int g = tid + gi * NT;
      if (g < Kw) {
        float gn[16];
        if (a.gain) load_gain16(a.gain, (int64_t)g * 16, gn);
#pragma unroll
        for (int m = 0; m < MM; ++m)
          if (m < M) quant_group(g, m, vk[gi][m], gn);
      }
    }
  } else {
#pragma unroll 2
    for (int g = tid; g < Kw; g += NT) {
      float gn[16];
      if (a.gain) load_gain16(a.gain, (int64_t)g * 16, gn);
#pragma unroll
      for (int m = 0; m < MM; ++m) {
        if (m < M) {
          float v[16];
          load_x(m, g, v);
          quant_group(g, m, v, gn);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    if (m < M) {
      const int t = warp_sum_i(rs[m]);
      if (lane == 0) red_i[warp * kMaxTok + m] = t;
    }
  }
  consumer_sync();

  // ------------------------------------------------------------- main loop
  // A stage holds RS whole rows (of each matrix).  Work items are (block of
  // RB rows, K-slice) pairs, WK slices per block, dealt round robin to the
  // consumer warps and continuing from stage to stage, so the load evens out
  // over the whole op and no stage waits for all warps.  With one slice per
  // block (WK == 1) the warp that reduces a block finishes its outputs from
  // registers.  Otherwise every slice adds its per-row totals into exact
  // integer accumulators in shared memory (one set per ring stage), and the
  // warp that completes a block's last slice (per-block counter) finishes
  // the block's outputs and clears the accumulators.
  const uint32_t x_addr = smem_u32(xperm);
  const int cnt_words = (int)sm.cnt_words;
  // dequantise and store one output (row `rr` of the current stage, token m)
  auto finish = [&](int r0, int rr, int m, int v0, int v1) {
    const int n = r0 + rr;
    const int64_t oo = (int64_t)m * N + n;
    // the token's row sum, from the per-warp partials (stable until the
    // kernel ends)
    int rsum = 0;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) rsum += red_i[w * kMaxTok + m];
    if constexpr (MODE == kGlu) {
      const int ag = v0 - rsum, au = v1 - rsum;
      const float g = __fmul_rn(__int2float_rn(ag), tok_d0[m]);
      const float u = __fmul_rn(__int2float_rn(au), tok_d1[m]);
      const float rg = fmaxf(g, 0.0f);
      a.h[oo] = __fmul_rn(__fmul_rn(rg, rg), u);
      if (a.acc0) a.acc0[oo] = ag;
      if (a.acc1) a.acc1[oo] = au;
    } else {
      const int ac = v0 - rsum;
      float y32 = __fmul_rn(__int2float_rn(ac), tok_d0[m]);
      if (MODE == kDown) y32 = __fmul_rn(y32, tok_f[m]);
      a.y[oo] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
      if (a.y_f32) a.y_f32[oo] = y32;
      if (a.acc0) a.acc0[oo] = ac;
    }
  };
  int base = 0;   // the warp that takes item 0 of the current stage
  for (int c = 0; c < nchunks; ++c) {
    const int s = gs;
    const uint32_t ph = gph;
    if (++gs == S) { gs = 0; gph ^= 1u; }
    const int r0 = n0 + c * RS;
    const int nr = min(RS, n1 - r0);
    const int nitems = ((nr + RB - 1) / RB) * WK;
    int first = warp - base;
    if (first < 0) first += kConsumerWarps;
    base = (base + nitems) % kConsumerWarps;
    // every warp waits for the stage's data before it releases the stage,
    // also with no item in it: an early release could count towards the
    // previous use of the stage, which slower warps may still be reading
    if (ring_ok && !mbar_wait(&sm.full()[s], ph)) ring_ok = false;
    if (first < nitems && ring_ok) {
      const uint32_t st_addr = smem_u32(sm.ring() + (size_t)s * sm.stage_bytes);
      int* acc = sm.acc_s() + s * acc_words;
      int* cnt = sm.cnt_s() + s * cnt_words;
      if constexpr (kMma) {
      // Tensor-core items: a 16-row tile (per matrix) x a K-slice of 16-word
      // windows.  MMA row = tile row, MMA k = activation position, MMA
      // column = token.  Lane (g = lane/4, q = lane%4) loads words 4q..4q+3
      // of rows g and g+8 of each window (16 bytes each) and the four
      // 16-activation groups of those words for token g.  Word 4q+2p gives
      // k = 4q..4q+3 and word 4q+2p+1 gives k = 16+4q..16+4q+3 of the MMA
      // for pair p and code plane t (masked in place, so its codes are
      // scaled by 4^t; one accumulator set per plane, shifted back at the
      // end, exactly).
      const int g = lane >> 2, qd = lane & 3;
      const int nwin = (Kw + 15) >> 4;
      const uint32_t xa = x_addr + (uint32_t)(g * K + 64 * qd);
      const bool tok_ok = g < M;
      for (int it = first; it < nitems; it += kConsumerWarps) {
        const int b = it >> wk_log2, q = it & (WK - 1);
        const int w0 = (q * nwin) >> wk_log2, w1 = ((q + 1) * nwin) >> wk_log2;
        uint32_t rowa[NMAT][2];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            rowa[mat][h] = st_addr + (uint32_t)((mat * RS + 16 * b + g + 8 * h) * Kb + 16 * qd);
        int C[NMAT][4][4];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
          for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) C[mat][t][e] = 0;
        for (int w = w0; w < w1; ++w) {
          // the row's last window may be partial: lanes past the end add 0
          const bool valid = 16 * w + 4 * qd < Kw;
          uint4 wr[NMAT][2];
#pragma unroll
          for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              wr[mat][h] = valid ? lds_v4(rowa[mat][h] + 64u * w) : make_uint4(0, 0, 0, 0);
          uint4 xg[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            xg[i] = (valid && tok_ok) ? lds_v4(xa + 256u * w + 16u * i) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint32_t mask = 0x03030303u << (2 * t);
              const uint32_t b0 = u4_at(xg[2 * pp], t), b1 = u4_at(xg[2 * pp + 1], t);
#pragma unroll
              for (int mat = 0; mat < NMAT; ++mat)
                mma_u8s8(C[mat][t], u4_at(wr[mat][0], 2 * pp) & mask,
                         u4_at(wr[mat][1], 2 * pp) & mask, u4_at(wr[mat][0], 2 * pp + 1) & mask,
                         u4_at(wr[mat][1], 2 * pp + 1) & mask, b0, b1);
            }
          }
        }
        // C element e: row g + 8*(e/2) of the tile, token 2q + e%2
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int v[NMAT];
#pragma unroll
          for (int mat = 0; mat < NMAT; ++mat)
            v[mat] = C[mat][0][e] + (C[mat][1][e] >> 2) + (C[mat][2][e] >> 4) + (C[mat][3][e] >> 6);
          const int rr = 16 * b + g + 8 * (e >> 1), m = 2 * qd + (e & 1);
          if (m < M && rr < nr) {
            if (WK == 1) {
              finish(r0, rr, m, v[0], v[NMAT - 1]);
            } else {
#pragma unroll
              for (int mat = 0; mat < NMAT; ++mat)
                atomicAdd(&acc[(mat * RS + rr) * kMaxTok + m], v[mat]);
            }
          }
        }
        if (WK > 1) {
          // the warp that adds a block's last slice finishes the block
          __syncwarp();
          int last = 0;
          if (lane == 0) {
            __threadfence_block();
            last = atomicAdd(&cnt[b], 1) == WK - 1;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence_block();
            const int rows_b = min(RB, nr - RB * b);
            for (int o = lane; o < rows_b * M; o += 32) {
              const int rr = RB * b + o / M, m = o % M;
              int* p0 = &acc[rr * kMaxTok + m];
              const int v0 = *p0;
              *p0 = 0;
              int v1 = 0;
              if (NMAT == 2) {
                int* p1 = &acc[(RS + rr) * kMaxTok + m];
                v1 = *p1;
                *p1 = 0;
              }
              finish(r0, rr, m, v0, v1);
            }
            if (lane == 0) cnt[b] = 0;
          }
        }
      }
      } else {
      for (int it = first; it < nitems; it += kConsumerWarps) {
        const int b = it >> wk_log2, q = it & (WK - 1);
        const int j0 = (q * Kw) >> wk_log2, j1 = ((q + 1) * Kw) >> wk_log2;
        uint32_t rowa[NR];             // shared-window byte address of each row
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          const int row = (NMAT == 2) ? (r >> 1) : r;
          const int mat = (NMAT == 2) ? (r & 1) : 0;
          rowa[r] = st_addr + (uint32_t)((mat * RS + RB * b + row) * Kb);
        }
        for (int tg = 0; tg < M; tg += MT) {
          int acc_r[NR][MT];
          int acc4[NR][4];   // MT == 1: one accumulator per code plane
#pragma unroll
          for (int r = 0; r < NR; ++r) {
#pragma unroll
            for (int t = 0; t < MT; ++t) acc_r[r][t] = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) acc4[r][p] = 0;
          }
          const uint32_t xt_addr = x_addr + (uint32_t)(tg * K);
#pragma unroll 2
          for (int j = j0 + lane; j < j1; j += 32) {
            uint32_t w[NR];
#pragma unroll
            for (int r = 0; r < NR; ++r) w[r] = lds_u32(rowa[r] + 4u * j);
            uint4 xv[MT];
#pragma unroll
            for (int t = 0; t < MT; ++t) xv[t] = lds_v4(xt_addr + (uint32_t)(t * K) + 16u * j);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
              if constexpr (MT == 1) {
                acc4[r][0] = dp4a_su((int)xv[0].x, w[r] & 0x03030303u, acc4[r][0]);
                acc4[r][1] = dp4a_su((int)xv[0].y, w[r] & 0x0c0c0c0cu, acc4[r][1]);
                acc4[r][2] = dp4a_su((int)xv[0].z, w[r] & 0x30303030u, acc4[r][2]);
                acc4[r][3] = dp4a_su((int)xv[0].w, w[r] & 0xc0c0c0c0u, acc4[r][3]);
              } else {
                const uint32_t c0 = w[r] & 0x03030303u;
                const uint32_t c1 = (w[r] >> 2) & 0x03030303u;
                const uint32_t c2 = (w[r] >> 4) & 0x03030303u;
                const uint32_t c3 = (w[r] >> 6) & 0x03030303u;
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                  int v = acc_r[r][t];
                  v = dp4a_su((int)xv[t].x, c0, v);
                  v = dp4a_su((int)xv[t].y, c1, v);
                  v = dp4a_su((int)xv[t].z, c2, v);
                  v = dp4a_su((int)xv[t].w, c3, v);
                  acc_r[r][t] = v;
                }
              }
            }
          }
          if constexpr (MT == 1) {
#pragma unroll
            for (int r = 0; r < NR; ++r)
              acc_r[r][0] = acc4[r][0] + (acc4[r][1] >> 2) + (acc4[r][2] >> 4) + (acc4[r][3] >> 6);
          }
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            int v[NR];
#pragma unroll
            for (int r = 0; r < NR; ++r) v[r] = acc_r[r][t];
            int tot, row, mat;
            bool writer;
            if constexpr (NR == 4) {
              // butterfly over 4 values: lane l ends with row l >> 3
              int h2[2], h1[1];
              halve<4>(v, h2, 16, lane);
              halve<2>(h2, h1, 8, lane);
              tot = h1[0];
              tot += __shfl_xor_sync(0xffffffffu, tot, 4);
              tot += __shfl_xor_sync(0xffffffffu, tot, 2);
              tot += __shfl_xor_sync(0xffffffffu, tot, 1);
              row = lane >> 3; mat = 0; writer = (lane & 7) == 0;
            } else {
              // butterfly over 8 values: lane l ends with value l >> 2
              int h4[4], h2[2], h1[1];
              halve<8>(v, h4, 16, lane);
              halve<4>(h4, h2, 8, lane);
              halve<2>(h2, h1, 4, lane);
              tot = h1[0];
              tot += __shfl_xor_sync(0xffffffffu, tot, 2);
              tot += __shfl_xor_sync(0xffffffffu, tot, 1);
              const int vi = lane >> 2;
              row = (NMAT == 2) ? (vi >> 1) : vi;
              mat = (NMAT == 2) ? (vi & 1) : 0;
              writer = (lane & 3) == 0;
            }
            const int m = tg + t;
            const int rr = RB * b + row;
            if (WK == 1) {
              // the whole row is in this lane: finish it here (Glu: the up
              // total sits 4 lanes up)
              const int up = (NMAT == 2) ? __shfl_down_sync(0xffffffffu, tot, 4) : 0;
              if (writer && mat == 0 && m < M && rr < nr) finish(r0, rr, m, tot, up);
            } else if (writer && m < M && rr < nr) {
              atomicAdd(&acc[(mat * RS + rr) * kMaxTok + m], tot);
            }
          }
        }
        if (WK > 1) {
          // the warp that adds a block's last slice finishes the block
          __syncwarp();
          int last = 0;
          if (lane == 0) {
            __threadfence_block();
            last = atomicAdd(&cnt[b], 1) == WK - 1;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence_block();
            const int rows_b = min(RB, nr - RB * b);
            for (int o = lane; o < rows_b * M; o += 32) {
              const int rr = RB * b + o / M, m = o % M;
              int* p0 = &acc[rr * kMaxTok + m];
              const int v0 = *p0;
              *p0 = 0;
              int v1 = 0;
              if (NMAT == 2) {
                int* p1 = &acc[(RS + rr) * kMaxTok + m];
                v1 = *p1;
                *p1 = 0;
              }
              finish(r0, rr, m, v0, v1);
            }
            if (lane == 0) cnt[b] = 0;
          }
        }
      }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty()[s]);
  }
}

// K-slices per row block.  Items (block x slice) are dealt round robin over
// the warps for the whole op, but only the stages in the ring at one time
// can be worked on together; each item costs its 32-word steps plus a fixed
// overhead (reduction, and with slices the shared atomics and counter).
static int pick_wk(int rows_cta, int rs, int rb, int Kw, int stages, int nch) {
  const int blocks_stage = (rs + rb - 1) / rb;
  const int blocks_total = (rows_cta + rb - 1) / rb + (nch - 1);
  const int window = stages < nch ? stages : nch;
  int best = 1;
  double best_cost = 1e30;
  for (int wk = 1; wk <= 32; wk *= 2) {
    if (wk > 1 && Kw / wk < 8) break;
    int par = blocks_stage * wk * window;
    if (par > kConsumerWarps) par = kConsumerWarps;
    const double rounds = (double)((blocks_total * wk + par - 1) / par);
    const double iters = (double)((Kw / wk + 31) / 32);
    const double cost = rounds * (iters + (wk > 1 ? 3.0 : 2.0));
    if (cost < best_cost - 1e-9) { best_cost = cost; best = wk; }
  }
  return best;
}

// Rows per work block: 16 (tensor-core items) for 4 or more tokens where 16
// rows of every matrix fit a 64 KB stage (measured: 7 % faster at M = 4 and
// 8, slower at M = 1, where dp4a does one token's work only); else dp4a
// items of 8 rows for a single matrix with long rows and one token (the
// activation loads and the reduction are shared by more rows), or 4.
static int gemv_rows_per_block(int M, int K, int nmat) {
  if (M >= 4 && (size_t)16 * (K / 4) * nmat <= 64 * 1024) return 16;
  return (nmat == 1 && M == 1 && K >= 8192) ? 8 : 4;
}


template <int MODE, int MT, int MM>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  DecodeSmem sm;
  sm.S = p.stages;
  sm.stage_bytes = p.stage_bytes;
  sm.xbytes = p.xbytes;
  sm.acc_words = p.acc_words;
  sm.cnt_words = p.cnt_words;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < sm.S; ++s) {
      mbar_init(&sm.full()[s], 1);
      mbar_init(&sm.empty()[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) pdl_launch_dependents();

  if (warp == kConsumerWarps) {
    if (lane == 0) produce(p.op, sm);
    return;
  }

  {   // accumulators and block counters start (and stay, between uses) at zero
    const int n_acc = sm.S * (int)sm.acc_words, n_cnt = sm.S * (int)sm.cnt_words;
    for (int i = tid; i < n_acc; i += kConsumerWarps * 32) sm.acc_s()[i] = 0;
    for (int i = tid; i < n_cnt; i += kConsumerWarps * 32) sm.cnt_s()[i] = 0;
  }
  bool ring_ok = true;
  pdl_wait();
  // 16-row tiles: the tensor-core items (planned on the host for 4 or more
  // tokens; not compiled into the 1- and 2-token kernels)
  if constexpr (MM >= 4) {
    if (p.op.rb == 16) {
      run_op<MODE, MT, MM, 16>(p.op, p.M, sm, ring_ok);
      return;
    }
  }
  // 8-row blocks: one long-row matrix with one token (planned on the host)
  if constexpr (MM == 1 && MODE != kGlu) {
    if (p.op.rb == 8) {
      run_op<MODE, MT, MM, 8>(p.op, p.M, sm, ring_ok);
      return;
    }
  }
  run_op<MODE, MT, MM, 4>(p.op, p.M, sm, ring_ok);
}

template <int MODE, int MT, int MM>
static cudaError_t launch_decode(const DecodeParams& p, int grid, size_t smem,
                                 cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attr_once(configured, decode_kernel<MODE, MT, MM>, 227 * 1024);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<MODE, MT, MM>, p);
}

template <int MODE>
static cudaError_t launch_by_tokens(const DecodeParams& p, int grid, size_t smem,
                                    cudaStream_t stream) {
  if (p.M == 1) return launch_decode<MODE, 1, 1>(p, grid, smem, stream);
  if (p.M == 2) return launch_decode<MODE, 2, 2>(p, grid, smem, stream);
  if (p.M <= 4) return launch_decode<MODE, 4, 4>(p, grid, smem, stream);
  return launch_decode<MODE, 4, 8>(p, grid, smem, stream);
}

// Host-side planning of a launch: rows per stage (stages of at most 56 KB,
// as few as cover the CTA's rows, equally sized), the work-block height, the
// ring depth (as many stages as the 227 KB of shared memory hold, 2..8) and
// the K-slicing.
static bitnet_status plan_decode(DecodeParams& p, int num_sms, int* grid_out, size_t* smem_out) {
  DecodeOp& o = p.op;
  const int M = p.M;
  const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
  const int Mpad = ((M + MT - 1) / MT) * MT;
  const int blocks = (o.N + 3) / 4;
  const int grid = blocks < num_sms ? blocks : num_sms;
  const int nmat = o.mode == kGlu ? 2 : 1;
  const size_t row_bytes = (size_t)(o.K / 4) * nmat;
  const int rb = gemv_rows_per_block(M, o.K, nmat);
  const int rows_per_cta = (o.N + grid - 1) / grid;
  // stages of at most 56 KB (64 KB where one 16-row tile needs it)
  int rs_max = (int)((56 * 1024) / row_bytes) / rb * rb;
  if (rs_max < rb) rs_max = rb;
  const int nch = (rows_per_cta + rs_max - 1) / rs_max;
  int rs = (rows_per_cta + nch - 1) / nch;
  rs = (rs + rb - 1) / rb * rb;
  const size_t stage = (size_t)rs * row_bytes;
  const size_t xbytes = (((size_t)Mpad * o.K + 127) / 128) * 128;
  const size_t accw = (size_t)nmat * rs * kMaxTok;
  const size_t cntw = (size_t)(rs / rb);
  // per ring stage: the stage itself, its accumulators and block counters
  const size_t budget = 227 * 1024;
  const size_t head = 4096 + xbytes + 256;
  const size_t per_stage = stage + 4 * (accw + cntw);
  int st = budget > head + 2 * per_stage ? (int)((budget - head) / per_stage) : 2;
  if (st > 8) st = 8;
  if (st > nch) st = nch;
  if (st < 2) st = 2;
  o.rb = rb;
  o.rows_per_stage = rs;
  // an MMA item step is a 16-word window of 16 rows (about twice a dp4a
  // item's 32-word step of 4 rows in time): planned as 2 steps of Kw/16
  o.wk = rb == 16 ? pick_wk(rows_per_cta, rs, rb, o.K / 8, st, nch)
                  : pick_wk(rows_per_cta, rs, rb, o.K / 16, st, nch);
  p.stages = st;
  p.stage_bytes = (uint32_t)stage;
  p.xbytes = (uint32_t)xbytes;
  p.acc_words = (uint32_t)accw;
  p.cnt_words = (uint32_t)cntw;
  *grid_out = grid;
  const size_t acc_bytes = ((st * accw + 31) / 32) * 128;
  const size_t cnt_bytes = ((st * cntw + 31) / 32) * 128;
  *smem_out = 4096 + xbytes + acc_bytes + cnt_bytes + (size_t)st * stage;
  return *smem_out > 227 * 1024 ? BITNET_ERR_UNSUPPORTED : BITNET_OK;
}

}  // namespace bitnet

using namespace bitnet;

// One decode launch: a BitLinear (mode kLinear), or the FFN's gate/up (kGlu)
// or down (kDown) step.  M <= 8.
bitnet_status bitnet_decode_launch(const DecodeOp& op, int M, int num_sms, cudaStream_t stream) {
  if (M < 1 || M > kMaxTok) return BITNET_ERR_UNSUPPORTED;
  DecodeParams p{};
  p.op = op;
  p.M = M;
  int grid = 0;
  size_t smem = 0;
  const bitnet_status st = plan_decode(p, num_sms, &grid, &smem);
  if (st != BITNET_OK) return st;
  cudaError_t e = cudaErrorInvalidValue;
  if (op.mode == kLinear) e = launch_by_tokens<kLinear>(p, grid, smem, stream);
  else if (op.mode == kGlu) e = launch_by_tokens<kGlu>(p, grid, smem, stream);
  else if (op.mode == kDown) e = launch_by_tokens<kDown>(p, grid, smem, stream);
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
