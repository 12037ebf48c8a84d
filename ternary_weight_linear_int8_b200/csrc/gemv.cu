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
// Layout of work: one CTA per SM-slot owns a contiguous range of output rows;
// warp 8 is the producer (bulk copies of whole rows, a few stages ahead);
// warps 0..7 each take blocks of 4 rows, lane l reading words l, l+32, ... of
// each row, then a butterfly reduction across the warp leaves row r's total
// in lane 8r.
//
// Programmatic dependent launch: the producer starts streaming weights
// before griddepcontrol.wait, the consumers wait before reading activations.
#include "common.cuh"

namespace bitnet {

enum GemvMode : int { kLinear = 0, kGlu = 1, kDown = 2 };

struct GemvArgs {
  const uint8_t* w0;      // packed [N, K/4]   (Glu: gate)
  const float* gamma0;
  const uint8_t* w1;      // Glu: up
  const float* gamma1;
  int N, K, M;
  const void* x;          // Linear/Glu: bf16 [M,K]; Down: fp32 h' [M,K]
  const float* gain;      // optional [K] (RMSNorm weight)
  const uint16_t* xnorm;  // Down: block input x [M,H] (for r1)
  int H;
  float eps;
  uint16_t* y;            // Linear/Down [M,N]
  float* y_f32;           // optional [M,N]
  int32_t* acc0;          // optional [M,N]
  int32_t* acc1;          // optional [M,N] (Glu up)
  float* h;               // Glu output h' [M,N]
  int8_t* xq_dbg;         // optional natural-layout x_q [M,K], written by CTA 0
  int rows_per_stage;     // multiple of 4
  int stages;             // 2..8
  int wk;                 // K-slices per 4-row block
};

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxTok = 8;
constexpr uint32_t kCopyChunk = 4096;   // bytes per bulk copy (a multiple of 16)

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
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

__device__ __forceinline__ float load_src(const void* x, bool f32, int64_t idx) {
  if (f32) return static_cast<const float*>(x)[idx];
  return bf16_bits_to_float(static_cast<const uint16_t*>(x)[idx]);
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

template <int MODE, int MT, int MM, int RB>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const GemvArgs a) {
  // MM: token count rounded up to 1, 2, 4 or 8 (loops over tokens unroll to
  // MM, keeping the code small for single-token decode)
  constexpr int NMAT = (MODE == kGlu) ? 2 : 1;
  // RB: rows per work block (per matrix); NR values per lane per block
  constexpr int NR = RB * NMAT;
  static_assert(NR == 4 || NR == 8, "4 or 8 values per block");
  constexpr bool kF32Src = (MODE == kDown);
  constexpr int NT = kConsumerWarps * 32;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + 8;
  float* tok_s = reinterpret_cast<float*>(smem + 128);
  float* tok_d0 = tok_s + kMaxTok;
  float* tok_d1 = tok_d0 + kMaxTok;
  float* tok_f = tok_d1 + kMaxTok;
  int* tok_rs = reinterpret_cast<int*>(tok_f + kMaxTok);
  float* red_f = reinterpret_cast<float*>(smem + 512);          // [16 warps][8 tok]
  int* red_i = reinterpret_cast<int*>(smem + 1024);             // [16][8]
  double* red_d = reinterpret_cast<double*>(smem + 2048);       // [16][8][2]
  const int M = a.M, K = a.K, N = a.N;
  const int Mpad = ((M + MT - 1) / MT) * MT;
  const int RS = a.rows_per_stage, S = a.stages, WK = a.wk;   // WK is a power of two
  const int wk_log2 = __ffs(WK) - 1;
  uint8_t* xperm = smem + 4096;
  const int xbytes = ((Mpad * K + 127) / 128) * 128;
  // per-stage integer accumulators [2 parity][NMAT][RS][kMaxTok]
  int* acc_s = reinterpret_cast<int*>(xperm + xbytes);
  const int acc_words = NMAT * RS * kMaxTok;
  const int acc_bytes = ((2 * acc_words * 4 + 127) / 128) * 128;
  uint8_t* ring = xperm + xbytes + acc_bytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Kb = K >> 2;                   // bytes per packed row
  const int Kw = K >> 4;                   // 32-bit words per packed row
  const int n0 = (int)(((int64_t)blockIdx.x * N) / gridDim.x);
  const int n1 = (int)(((int64_t)(blockIdx.x + 1) * N) / gridDim.x);
  const int nchunks = (n1 - n0 + RS - 1) / RS;
  const int stage_bytes = RS * Kb * NMAT;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) pdl_launch_dependents();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % S;
        if (c >= S && !mbar_wait(&empty[s], ((c / S) - 1) & 1)) break;
        const int r0 = n0 + c * RS;
        const int nr = min(RS, n1 - r0);
        const uint32_t bytes = (uint32_t)nr * Kb;
        mbar_arrive_expect_tx(&full[s], bytes * NMAT);
        uint8_t* dst = ring + (size_t)s * stage_bytes;
        // several 4 KB copies per stage keep more requests in flight than
        // one large copy
        for (uint32_t off = 0; off < bytes; off += kCopyChunk) {
          const uint32_t nb = bytes - off < kCopyChunk ? bytes - off : kCopyChunk;
          bulk_g2s(dst + off, a.w0 + (int64_t)r0 * Kb + off, nb, &full[s], pol);
          if (NMAT == 2)
            bulk_g2s(dst + (size_t)RS * Kb + off, a.w1 + (int64_t)r0 * Kb + off, nb, &full[s], pol);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- prologue
  for (int i = tid; i < 2 * acc_words; i += NT) acc_s[i] = 0;
  pdl_wait();
  for (int i = M * K + tid * 16; i < Mpad * K; i += NT * 16)
    *reinterpret_cast<uint4*>(xperm + i) = make_uint4(0, 0, 0, 0);

  // pass 1: per-token absmax of src*gain (and, for Down, sums of squares).
  // With one or two tokens and at most KEEPG groups of 16 per thread the
  // values stay in registers for pass 2 instead of being loaded again.
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
            load_group16<kF32Src>(a.x, (int64_t)m * K + g * 16, vk[gi][m]);
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
          load_group16<kF32Src>(a.x, (int64_t)m * K + g * 16, v);
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
    tok_d0[m] = __fdiv_rn(*a.gamma0, s);
    if (MODE == kGlu) tok_d1[m] = __fdiv_rn(*a.gamma1, s);
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
          load_group16<kF32Src>(a.x, (int64_t)m * K + g * 16, v);
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
  // the epilogue reads the row sums straight from the per-warp partials
  if (tid < M) {
    int t = 0;
    for (int w = 0; w < kConsumerWarps; ++w) t += red_i[w * kMaxTok + tid];
    tok_rs[tid] = t;
  }

  // ------------------------------------------------------------- main loop
  // A stage holds RS whole rows (of each matrix).  Work items are (block of
  // 4 rows, K-slice) pairs, WK slices per block, dealt to the 8 warps round
  // robin; each item's per-row totals are added into shared-memory integer
  // accumulators (exact, order-free), and after a barrier the stage's
  // outputs are finished from them.
  const uint32_t x_addr = smem_u32(xperm);
  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    const int s = c % S;
    if (ok && !mbar_wait(&full[s], (c / S) & 1)) ok = false;
    const int r0 = n0 + c * RS;
    const int nr = min(RS, n1 - r0);
    int* acc = acc_s + (c & 1) * acc_words;
    if (ok) {
      const uint32_t st_addr = smem_u32(ring + (size_t)s * stage_bytes);
      const int nitems = ((nr + RB - 1) / RB) * WK;
      for (int it = warp; it < nitems; it += kConsumerWarps) {
        const int b = it >> wk_log2, q = it & (WK - 1);
        const int j0 = (q * Kw) / WK, j1 = ((q + 1) * Kw) / WK;
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
            if (writer && m < M && RB * b + row < nr)
              atomicAdd(&acc[(mat * RS + RB * b + row) * kMaxTok + m], tot);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    consumer_sync();
    // finish this stage's outputs; clear the accumulators for stage c + 2
    for (int o = tid; o < nr * M; o += NT) {
      const int row = o / M, m = o - row * M;
      const int n = r0 + row;
      const int64_t oo = (int64_t)m * N + n;
      const int rsum = tok_rs[m];
      int* p0 = &acc[row * kMaxTok + m];
      if (MODE == kGlu) {
        int* p1 = &acc[(RS + row) * kMaxTok + m];
        const int ag = *p0 - rsum, au = *p1 - rsum;
        *p0 = 0;
        *p1 = 0;
        const float g = __fmul_rn(__int2float_rn(ag), tok_d0[m]);
        const float u = __fmul_rn(__int2float_rn(au), tok_d1[m]);
        const float rg = fmaxf(g, 0.0f);
        if (ok) a.h[oo] = __fmul_rn(__fmul_rn(rg, rg), u);
        if (ok && a.acc0) a.acc0[oo] = ag;
        if (ok && a.acc1) a.acc1[oo] = au;
      } else {
        const int ac = *p0 - rsum;
        *p0 = 0;
        float y32 = __fmul_rn(__int2float_rn(ac), tok_d0[m]);
        if (MODE == kDown) y32 = __fmul_rn(y32, tok_f[m]);
        if (ok) {
          a.y[oo] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
          if (a.y_f32) a.y_f32[oo] = y32;
          if (a.acc0) a.acc0[oo] = ac;
        }
      }
    }
  }
}

template <int MODE, int MT, int MM, int RB>
static cudaError_t launch_one(const GemvArgs& a, int grid, size_t smem, cudaStream_t stream) {
  static unsigned long long configured = 0;   // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured & (1ull << (dev & 63)))) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<MODE, MT, MM, RB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    configured |= 1ull << (dev & 63);
  }
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
  return cudaLaunchKernelEx(&cfg, gemv_kernel<MODE, MT, MM, RB>, a);
}

// Host-side planning: stage rows and ring depth under a shared-memory budget
// that leaves room for a second CTA per SM (the next kernel in the stream).
struct GemvPlan {
  int grid, rows_per_stage, stages, wk;
  size_t smem;
};

// K-slices per row block: balance (blocks x slices) items over the warps
// against the fixed cost of an item (reduction, shared atomics, set-up).
static int pick_wk(int nb, int Kw) {
  int best = 1;
  double best_cost = 1e30;
  for (int wk = 1; wk <= 32; wk *= 2) {
    if (wk > 1 && Kw / wk < 8) break;
    const double rounds = (double)((nb * wk + kConsumerWarps - 1) / kConsumerWarps);
    const double iters = (double)((Kw / wk + 31) / 32);
    const double cost = rounds * (iters + 2.0);   // per-item reduction ~ two 32-word steps
    if (cost < best_cost - 1e-9) { best_cost = cost; best = wk; }
  }
  return best;
}

// Rows per work block: 8 for a single matrix with long rows and one token
// (the activation loads and the reduction are shared by more rows), else 4.
static int gemv_rows_per_block(int M, int K, int nmat) {
  return (nmat == 1 && M == 1 && K >= 8192) ? 8 : 4;
}

static GemvPlan plan_gemv(int M, int N, int K, int nmat, int num_sms, int MT) {
  GemvPlan p{};
  const int Mpad = ((M + MT - 1) / MT) * MT;
  const size_t xbytes = (((size_t)Mpad * K + 127) / 128) * 128;
  const size_t budget = 200 * 1024;
  const size_t row_bytes = (size_t)(K / 4) * nmat;
  int blocks = (N + 3) / 4;
  p.grid = blocks < num_sms ? blocks : num_sms;
  const int rows_per_cta = (N + p.grid - 1) / p.grid;
  // stages of at most 56 KB, as few as cover the CTA's rows, equally sized
  const int rb = gemv_rows_per_block(M, K, nmat);
  int rs_max = (int)((56 * 1024) / row_bytes) / rb * rb;
  if (rs_max < rb) rs_max = rb;
  const int nch = (rows_per_cta + rs_max - 1) / rs_max;
  int rs = (rows_per_cta + nch - 1) / nch;
  rs = (rs + rb - 1) / rb * rb;
  const size_t acc_bytes = ((2 * (size_t)nmat * rs * kMaxTok * 4 + 127) / 128) * 128;
  const size_t head = 4096 + xbytes + acc_bytes;
  const size_t ring = budget > head + 2 * (size_t)rs * row_bytes ? budget - head
                                                                  : 2 * (size_t)rs * row_bytes;
  int st = (int)(ring / ((size_t)rs * row_bytes));
  if (st > 8) st = 8;
  if (st < 2) st = 2;
  if (st > nch) st = nch < 2 ? 2 : nch;
  p.rows_per_stage = rs;
  p.stages = st;
  p.wk = pick_wk(rs / rb, K / 16);
  p.smem = head + (size_t)st * rs * row_bytes;
  return p;
}

}  // namespace bitnet

using namespace bitnet;

size_t bitnet_gemv_smem_bytes(int M, int N, int K, int nmat, int num_sms) {
  const int MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
  return plan_gemv(M, N, K, nmat, num_sms, MT).smem;
}

bitnet_status bitnet_gemv_launch(int mode, GemvArgs a, int num_sms, cudaStream_t stream) {
  const int nmat = mode == kGlu ? 2 : 1;
  const int MT = a.M == 1 ? 1 : (a.M == 2 ? 2 : 4);
  const GemvPlan p = plan_gemv(a.M, a.N, a.K, nmat, num_sms, MT);
  if (p.smem > 227 * 1024) return BITNET_ERR_UNSUPPORTED;
  a.rows_per_stage = p.rows_per_stage;
  a.stages = p.stages;
  a.wk = p.wk;
  const int rb = gemv_rows_per_block(a.M, a.K, nmat);
  cudaError_t e = cudaErrorInvalidValue;
#define BITNET_GEMV_CASE(MODE_)                                                       \
  if (mode == MODE_) {                                                                \
    if (a.M == 1 && rb == 8) e = launch_one<MODE_, 1, 1, (MODE_ == kGlu ? 4 : 8)>(a, p.grid, p.smem, stream); \
    else if (a.M == 1) e = launch_one<MODE_, 1, 1, 4>(a, p.grid, p.smem, stream);     \
    else if (a.M == 2) e = launch_one<MODE_, 2, 2, 4>(a, p.grid, p.smem, stream);     \
    else if (a.M <= 4) e = launch_one<MODE_, 4, 4, 4>(a, p.grid, p.smem, stream);     \
    else e = launch_one<MODE_, 4, 8, 4>(a, p.grid, p.smem, stream);                   \
  }
  BITNET_GEMV_CASE(kLinear)
  BITNET_GEMV_CASE(kGlu)
  BITNET_GEMV_CASE(kDown)
#undef BITNET_GEMV_CASE
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
