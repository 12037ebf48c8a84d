// Resident decode kernel: BitLinear for a few tokens on layers whose
// per-CTA slice of packed weights fits in shared memory next to the
// quantised activations (2B-class decode: about 30 KB of weights per SM).
//
// dashen-tech.com "BitNet.cpp 深度解析", section "3.1 計算コア：整数行列乗算":
// the product with ternary weights is sum_pos - sum_neg, taken here in the
// offset form sum_k x_q * code - sum_k x_q (code = w + 1) with dp4a on the
// masked code planes of each packed word, exactly as the streaming decode
// kernel does.
//
// What differs from the streaming decode kernel is the schedule.  Two CTAs
// fit on each SM (at most 112 KB of shared memory and 64 registers per
// thread), so with programmatic dependent launch the CTA of the next layer
// becomes resident while this layer computes.  Its first act is to request
// its whole weight slice with bulk async copies (before griddepcontrol.wait:
// weights never depend on the previous kernel), so in a chain of layers the
// weights land while the layers before finish, and after the wait only the
// dependent sequence remains: activation loads, per-token absmax and
// quantisation into shared memory, the products from shared memory and the
// dequantised stores.
//
// Two more weight formats share the schedule (template parameter FMT):
//  * kResW1 -- BitNet v1 sign weights, one bit each (youngju.dev page,
//    section "BitNet v1：BitLinearの誕生" > "1-Bit重みとSign関数"): bit 1 for
//    +1, 0 for -1, 8 weights per byte along K, least significant bit first.
//    Plane p of a 32-bit word, (w >> p) & 0x01010101, holds in byte b the bit
//    of k = 32j + 8b + p, and the activations sit in the matching order (in
//    each group of 32, slot 4p + b holds k = 8b + p), so dp4a gives the sum
//    of x over the +1 weights, S; then x . W_b = 2 S - sum x.
//  * kResTL2 -- the ternary I2_S weights through pair lookup tables instead
//    of dp4a (the TL2 idea of the youngju.dev page, section
//    "I2_Sカーネルの内部動作": two ternary weights index one table entry).  For
//    every activation pair (x0, x1) = (x_q[2i], x_q[2i+1]) a 16-entry table
//    holds x0 (c0 - 1) + x1 (c1 - 1) at c0 + 4 c1; a packed nibble is exactly
//    that index, so a byte costs two lookups.  One token; one CTA per SM (the
//    tables take 16 K bytes).
//  * kResA48 -- the ternary I2_S weights on one token in BitNet a4.8 form
//    (youngju.dev page, section "BitNet a4.8：ハイブリッド量子化戦略"): the
//    token becomes two code rows in the kernel order, the 4-bit codes of the
//    ordinary values and the 8-bit codes of the largest ones, with their
//    scales and row sums -- computed by every CTA from the bf16 token in its
//    prologue (the a4.8 selection, the same in every CTA), or given already
//    quantised; the dp4a items run on both rows and the epilogue forms
//    fp32(acc4) (gamma / s4) + fp32(acc8) (gamma / s8).
#include "common.cuh"

namespace bitnet {

enum ResFmt : int { kResI2S = 0, kResW1 = 1, kResTL2 = 2, kResA48 = 3 };

struct ResidentParams {
  const uint8_t* w;        // packed [N, K/4] (I2_S) or [N, K/8] (sign bits)
  const float* gamma;      // gamma (I2_S) or alpha (sign weights)
  const uint16_t* x;       // bf16 [M, K]
  uint16_t* y;             // bf16 [M, N]
  float* y_f32;            // optional [M, N]
  int32_t* acc;            // optional [M, N]
  int N, K, M;
  int wk;                  // K-slices per 4-row block (1, 2, 4 or 8)
  int pieces;              // weight copy groups (1..4), one mbarrier each
  uint32_t x_off;          // shared-memory offsets (bytes, multiples of 128)
  uint32_t lut_off;        // pair tables (kResTL2)
  uint32_t acc_off;
  uint32_t w_off;
  const int8_t* xq_in;     // kResA48: code rows [2][K] (kernel order), or null:
                           // quantise x with n_out 8-bit values in the prologue
  int n_out;
  const float* s_in;       // kResA48: their scales [2]
  const int32_t* rs_in;    // kResA48: their row sums [2]
  int32_t* acc8;           // kResA48: optional [N] (acc holds acc4)
};

constexpr int kResWarps = 16;
constexpr int kResThreads = kResWarps * 32;
constexpr int kResMaxTok = 8;
// two CTAs per SM: 228 KB of shared memory per SM, 1 KB reserved per CTA;
// the pair tables need one CTA per SM
__host__ __device__ constexpr uint32_t res_smem_max(int fmt) {
  return fmt == kResTL2 ? 200u * 1024u : 112u * 1024u;
}
constexpr uint32_t kResHead = 1152;     // barriers, token scalars, warp partials

extern __shared__ __align__(128) uint8_t g_res_smem[];

// MT: tokens per dp4a pass; MM: token count rounded up (loop bound).
template <int FMT, int MT, int MM>
__global__ void __launch_bounds__(kResThreads, FMT == kResTL2 ? 1 : 2)
    resident_kernel(const __grid_constant__ ResidentParams p) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(g_res_smem);          // [4]
  float* tok_d = reinterpret_cast<float*>(g_res_smem + 64);          // [8]
  float* red_f = reinterpret_cast<float*>(g_res_smem + 128);         // [16 warps][8]
  int* red_i = reinterpret_cast<int*>(g_res_smem + 640);             // [16 warps][8]
  uint8_t* xq = g_res_smem + p.x_off;                                // [Mpad][K]
  int* accs = reinterpret_cast<int*>(g_res_smem + p.acc_off);        // [rows][8] (wk > 1)
  uint8_t* wsm = g_res_smem + p.w_off;                               // [rows][Rb]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, N = p.N, M = p.M;
  const int Rb = FMT == kResW1 ? K >> 3 : K >> 2;   // packed bytes per row
  const int Ww = FMT == kResW1 ? K >> 5 : K >> 4;   // 32-bit words per row
  const int n0 = (int)(((int64_t)blockIdx.x * N) / gridDim.x);
  const int n1 = (int)(((int64_t)(blockIdx.x + 1) * N) / gridDim.x);
  const int R = n1 - n0;
  const int nblk = (R + 3) >> 2;       // 4-row blocks
  const int P = p.pieces;
  const int cs = (nblk + P - 1) / P;   // blocks per piece

  // ---- weights: the whole slice, in P pieces of cs whole 4-row blocks
  if (tid == 0) {
    for (int i = 0; i < P; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    pdl_launch_dependents();
    const uint64_t pol = policy_evict_first();
    for (int i = 0; i < P; ++i) {
      const int r0 = min(R, 4 * i * cs);
      const int r1 = min(R, 4 * (i + 1) * cs);
      if (r1 <= r0) {            // empty piece: complete its phase at once
        mbar_arrive(&bars[i]);
        continue;
      }
      const uint32_t bytes = (uint32_t)(r1 - r0) * (uint32_t)Rb;
      mbar_arrive_expect_tx(&bars[i], bytes);
      const uint8_t* src = p.w + (int64_t)(n0 + r0) * Rb;
      uint8_t* dst = wsm + (size_t)r0 * Rb;
      for (uint32_t off = 0; off < bytes; off += 4096u) {
        const uint32_t nb = bytes - off < 4096u ? bytes - off : 4096u;
        bulk_g2s(dst + off, src + off, nb, &bars[i], pol);
      }
    }
  }
  // dp4a passes read MT tokens at a time: the padding tokens are zero
  const int Mpad = ((M + MT - 1) / MT) * MT;
  for (int i = M * K + tid * 16; i < Mpad * K; i += kResThreads * 16)
    sts_v4(smem_u32(xq + i), make_uint4(0, 0, 0, 0));
  const int WK = p.wk;
  if (WK > 1)
    for (int i = tid; i < nblk * 4 * kResMaxTok; i += kResThreads) accs[i] = 0;

  pdl_wait();

  int rtot[MM];
  if constexpr (FMT == kResA48) {
    static_assert(kResThreads == kA48Threads, "the a4.8 selection runs on the whole block");
    if (p.xq_in) {
      // the two code rows as they are, their dequant factors and row sums
      for (int i = tid * 16; i < M * K; i += kResThreads * 16)
        sts_v4(smem_u32(xq + i), *reinterpret_cast<const uint4*>(p.xq_in + i));
      if (tid < M) tok_d[tid] = __fdiv_rn(*p.gamma, p.s_in[tid]);
#pragma unroll
      for (int m = 0; m < MM; ++m) rtot[m] = m < M ? p.rs_in[m] : 0;
    } else {
      // the token's a4.8 selection and codes (identical in every CTA),
      // straight into the shared code rows
      const A48Token t = a48_quant_token(p.x, K, p.n_out, reinterpret_cast<int8_t*>(xq),
                                         reinterpret_cast<int8_t*>(xq + K), nullptr, nullptr);
      if (tid == 0) {
        tok_d[0] = __fdiv_rn(*p.gamma, t.s4);
        tok_d[1] = __fdiv_rn(*p.gamma, t.s8);
      }
      rtot[0] = t.rs4;
      rtot[MM - 1] = t.rs8;
    }
    __syncthreads();
  } else {
  // ---- per-token absmax (pass 1) and quantisation (pass 2).  A thread owns
  // (token, 8 consecutive values) pairs; up to two pairs per thread stay in
  // registers between the passes, otherwise pass 2 loads them again.
  float gam = 0.f;
  if (tid < M) gam = *p.gamma;
  const int Kh = K >> 3;                 // 8-value pieces per token
  const int npair = M * Kh;
  const bool keep = npair <= 2 * kResThreads;
  uint4 kv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  float am[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) am[m] = 0.f;
  auto absmax8 = [](const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
    }
    return mx;
  };
  auto tok_of = [&](int pi) { return MM == 1 ? 0 : pi / Kh; };
  if (keep) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int pi = tid + i * kResThreads;
      if (pi < npair) {
        const int m = tok_of(pi);
        kv[i] = *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + (pi - m * Kh) * 8);
        const float mx = absmax8(kv[i]);
#pragma unroll
        for (int mm = 0; mm < MM; ++mm)
          if (mm == m) am[mm] = fmaxf(am[mm], mx);
      }
    }
  } else {
    for (int pi = tid; pi < npair; pi += kResThreads) {
      const int m = tok_of(pi);
      const float mx =
          absmax8(*reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + (pi - m * Kh) * 8));
#pragma unroll
      for (int mm = 0; mm < MM; ++mm)
        if (mm == m) am[mm] = fmaxf(am[mm], mx);
    }
  }
  // warp maxima with one redux each (|x| >= 0, so the bit patterns order
  // like the values), then every warp reduces the warp maxima the same way
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(am[m]));
    if (lane == 0 && m < M) red_f[warp * kResMaxTok + m] = __uint_as_float(w);
  }
  __syncthreads();
  float sc[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const uint32_t v =
        (m < M && lane < kResWarps) ? __float_as_uint(red_f[lane * kResMaxTok + m]) : 0u;
    sc[m] = qscale(__uint_as_float(__reduce_max_sync(0xffffffffu, v)));
  }
  if (tid < M) {
    float s = sc[0];
#pragma unroll
    for (int mm = 1; mm < MM; ++mm)
      if (mm == tid) s = sc[mm];
    tok_d[tid] = __fdiv_rn(gam, s);
  }
  int rs[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) rs[m] = 0;
  auto quant8 = [&](int pi, const uint4& v) {
    const int m = tok_of(pi), hg = pi - m * Kh;
    float s = sc[0];
#pragma unroll
    for (int mm = 1; mm < MM; ++mm)
      if (mm == m) s = sc[mm];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    int q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      q[2 * i] = quant_code_sat(__uint_as_float(w[i] << 16), s);
      q[2 * i + 1] = quant_code_sat(__uint_as_float(w[i] & 0xffff0000u), s);
    }
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) sum += q[i];
    const uint32_t row = smem_u32(xq) + (uint32_t)(m * K);
    if constexpr (FMT == kResI2S) {
      // k = 16g + 8h + i lands at slot 4 (i % 4) + 2h + i / 4 of group g: per
      // code plane t one 16-bit half (values t and t + 4)
      const uint32_t base = row + (uint32_t)((hg >> 1) * 16 + 2 * (hg & 1));
#pragma unroll
      for (int t = 0; t < 4; ++t)
        sts_u16(base + 4 * t, (uint16_t)__byte_perm((uint32_t)q[t], (uint32_t)q[4 + t], 0x0040));
    } else if constexpr (FMT == kResW1) {
      // k = 32G + 8h + i lands at slot 4i + h of group G
      const uint32_t base = row + (uint32_t)((hg >> 2) * 32 + (hg & 3));
#pragma unroll
      for (int i = 0; i < 8; ++i) sts_u8(base + 4 * i, (uint8_t)q[i]);
    } else {
      // natural order (the pair tables are built from it)
      const uint32_t lo = __byte_perm(__byte_perm((uint32_t)q[0], (uint32_t)q[1], 0x0040),
                                      __byte_perm((uint32_t)q[2], (uint32_t)q[3], 0x0040), 0x5410);
      const uint32_t hi = __byte_perm(__byte_perm((uint32_t)q[4], (uint32_t)q[5], 0x0040),
                                      __byte_perm((uint32_t)q[6], (uint32_t)q[7], 0x0040), 0x5410);
      sts_v2(row + (uint32_t)(hg * 8), lo, hi);
    }
#pragma unroll
    for (int mm = 0; mm < MM; ++mm)
      if (mm == m) rs[mm] += sum;
  };
  if (keep) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int pi = tid + i * kResThreads;
      if (pi < npair) quant8(pi, kv[i]);
    }
  } else {
    for (int pi = tid; pi < npair; pi += kResThreads) {
      const int m = tok_of(pi);
      quant8(pi, *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + (pi - m * Kh) * 8));
    }
  }
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const int t = __reduce_add_sync(0xffffffffu, rs[m]);
    if (lane == 0 && m < M) red_i[warp * kResMaxTok + m] = t;
  }
  __syncthreads();
  if constexpr (FMT == kResTL2) {
    // pair tables: entry c0 + 4 c1 of pair i is x0 (c0 - 1) + x1 (c1 - 1)
    // (code 3 never occurs; its entries are 0); 16 int16 = 32 bytes a pair
    const uint32_t lut = smem_u32(g_res_smem + p.lut_off);
    for (int pr = tid; pr < (K >> 1); pr += kResThreads) {
      const int x0 = (int)(int8_t)xq[2 * pr], x1 = (int)(int8_t)xq[2 * pr + 1];
      uint32_t e[8];
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) {
        int v2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int idx = 2 * w2 + h, c0 = idx & 3, c1 = idx >> 2;
          v2[h] = (c0 == 3 || c1 == 3) ? 0 : x0 * (c0 - 1) + x1 * (c1 - 1);
        }
        e[w2] = ((uint32_t)v2[0] & 0xffffu) | ((uint32_t)v2[1] << 16);
      }
      sts_v4(lut + 32u * pr, make_uint4(e[0], e[1], e[2], e[3]));
      sts_v4(lut + 32u * pr + 16u, make_uint4(e[4], e[5], e[6], e[7]));
    }
    __syncthreads();
  }
  // each token's row sum (identical in every thread)
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    const int v = (m < M && lane < kResWarps) ? red_i[lane * kResMaxTok + m] : 0;
    rtot[m] = __reduce_add_sync(0xffffffffu, v);
  }
  }

  // ---- products: items (4-row block b, K-slice q), dealt round robin to the
  // warps; lane l reads words l, l+32, ... of the slice of each row.
  auto finish = [&](int r, int m, int v) {
    int rsum = rtot[0];
#pragma unroll
    for (int mm = 1; mm < MM; ++mm)
      if (mm == m) rsum = rtot[mm];
    const int ac = FMT == kResTL2 ? v : (FMT == kResW1 ? 2 * v - rsum : v - rsum);
    const float y32 = __fmul_rn(__int2float_rn(ac), tok_d[m]);
    const int64_t o = (int64_t)m * N + n0 + r;
    p.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
    if (p.y_f32) p.y_f32[o] = y32;
    if (p.acc) p.acc[o] = ac;
  };
  // kResA48: one token from its two code rows (4-bit, then 8-bit), the two
  // fp32 products added in that order
  auto finish_a48 = [&](int r, int v4, int v8) {
    const int a4 = v4 - rtot[0], a8 = v8 - rtot[MM > 1 ? 1 : 0];
    const float y32 = __fadd_rn(__fmul_rn(__int2float_rn(a4), tok_d[0]),
                                __fmul_rn(__int2float_rn(a8), tok_d[1]));
    const int64_t o = n0 + r;
    p.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
    if (p.y_f32) p.y_f32[o] = y32;
    if (p.acc) p.acc[o] = a4;
    if (p.acc8) p.acc8[o] = a8;
  };
  const uint32_t x_addr = smem_u32(xq), w_addr = smem_u32(wsm);
  const uint32_t lut_addr = smem_u32(g_res_smem + p.lut_off);
  bool ok = true;
  int pc = 0;            // weight piece of the current block (blocks only grow)
  constexpr bool kTern = FMT == kResI2S || FMT == kResA48;   // I2_S codes, dp4a
  constexpr int kUnroll = (MT == 1 && kTern) ? 1 : 2;
  const int wkl = __ffs(WK) - 1;
  const int nitems = nblk * WK;
  for (int it = warp; it < nitems; it += kResWarps) {
    const int b = it >> wkl, qs = it & (WK - 1);
    while ((pc + 1) * cs <= b) ++pc;
    if (!mbar_wait(&bars[pc], 0)) { ok = false; break; }
    const int j0 = (qs * Ww) >> wkl, j1 = ((qs + 1) * Ww) >> wkl;
    uint32_t rowa[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) rowa[r] = w_addr + (uint32_t)(min(4 * b + r, R - 1) * Rb);
    for (int tg = 0; tg < M; tg += MT) {
      int acc_r[4][MT];
      int acc4[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int t = 0; t < MT; ++t) acc_r[r][t] = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) acc4[r][t] = 0;
      }
      const uint32_t xt = x_addr + (uint32_t)(tg * K);
#pragma unroll kUnroll
      for (int j = j0 + lane; j < j1; j += 32) {
        uint32_t w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) w[r] = lds_u32(rowa[r] + 4u * j);
        if constexpr (kTern) {
          uint4 xv[MT];
#pragma unroll
          for (int t = 0; t < MT; ++t) xv[t] = lds_v4(xt + (uint32_t)(t * K) + 16u * j);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
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
        } else if constexpr (FMT == kResW1) {
          // 32 activations per word: planes p = 0..7 against words p of the group
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const uint4 xa = lds_v4(xt + (uint32_t)(t * K) + 32u * j);
            const uint4 xb = lds_v4(xt + (uint32_t)(t * K) + 32u * j + 16u);
            const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              int v = acc_r[r][t];
#pragma unroll
              for (int pl = 0; pl < 8; ++pl)
                v = dp4a_su((int)xw[pl], (w[r] >> pl) & 0x01010101u, v);
              acc_r[r][t] = v;
            }
          }
        } else {
          // pair tables: byte q of the word holds pairs 2q (low nibble) and
          // 2q + 1 (high nibble) of this word's 8 pairs
          const uint32_t tb = lut_addr + 256u * (uint32_t)j;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            int v = acc_r[r][0];
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2) {
              const uint32_t nib = (w[r] >> (4 * q2)) & 15u;
              v += lds_s16(tb + 32u * q2 + 2u * nib);
            }
            acc_r[r][0] = v;
          }
        }
      }
      if constexpr (MT == 1 && kTern) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
          acc_r[r][0] = acc4[r][0] + (acc4[r][1] >> 2) + (acc4[r][2] >> 4) + (acc4[r][3] >> 6);
      }
      int tots[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int v[4] = {acc_r[0][t], acc_r[1][t], acc_r[2][t], acc_r[3][t]};
        // butterfly over the 4 rows: lane l ends with row l >> 3
        int h2[2], h1[1];
        halve<4>(v, h2, 16, lane);
        halve<2>(h2, h1, 8, lane);
        int tot = h1[0];
        tot += __shfl_xor_sync(0xffffffffu, tot, 4);
        tot += __shfl_xor_sync(0xffffffffu, tot, 2);
        tot += __shfl_xor_sync(0xffffffffu, tot, 1);
        tots[t] = tot;
        const int r = 4 * b + (lane >> 3), m = tg + t;
        if ((lane & 7) == 0 && m < M && r < R) {
          if (WK > 1) atomicAdd(&accs[r * kResMaxTok + m], tot);
          else if constexpr (FMT != kResA48) finish(r, m, tot);
        }
      }
      if constexpr (FMT == kResA48) {
        const int r = 4 * b + (lane >> 3);
        if (WK == 1 && (lane & 7) == 0 && r < R) finish_a48(r, tots[0], tots[MT - 1]);
      }
    }
  }
  if (WK > 1) {
    __syncthreads();
    if constexpr (FMT == kResA48) {
      for (int r = tid; r < R; r += kResThreads)
        finish_a48(r, accs[r * kResMaxTok], accs[r * kResMaxTok + 1]);
    } else {
      for (int o = tid; o < R * M; o += kResThreads) {
        const int r = MM == 1 ? o : o / M, m = o - r * M;
        finish(r, m, accs[r * kResMaxTok + m]);
      }
    }
  }
  if (!ok) {
    // a wait gave up (recorded in the status word): let this CTA's copies
    // finish, within the same limit, before its shared memory is released
    for (int i = 0; i < P; ++i) mbar_wait(&bars[i], 0);
  }
}

// Host-side plan: does the layer fit, and with how many K-slices and pieces.
struct ResidentPlan {
  ResidentParams p;
  int grid;
  uint32_t smem;
};

static uint32_t al128(uint64_t v) { return (uint32_t)((v + 127) & ~uint64_t(127)); }

static bool plan_resident(int fmt, int M, int N, int K, int num_sms, ResidentPlan* out) {
  if (M < 1 || M > (fmt == kResTL2 ? 1 : 3) || K % 64 != 0 || N < 1) return false;
  if (fmt == kResW1 && K % 128 != 0) return false;   // 16-byte packed rows
  const int MT = M == 1 ? 1 : 2;
  const int Mpad = ((M + MT - 1) / MT) * MT;
  const int grid = (N + 3) / 4 < num_sms ? (N + 3) / 4 : num_sms;
  const int rows_max = (N + grid - 1) / grid;
  const int nblk = (rows_max + 3) / 4;
  const int Ww = fmt == kResW1 ? K / 32 : K / 16;
  const int Rb = fmt == kResW1 ? K / 8 : K / 4;
  // K-slices: rounds of items over the warps x (32-word steps + a fixed
  // per-item cost of about two steps)
  int wk = 1;
  double best = 1e30;
  for (int c = 1; c <= 8; c *= 2) {
    if (c > 1 && Ww / c < 32) break;
    const double rounds = (double)((nblk * c + kResWarps - 1) / kResWarps);
    const double cost = rounds * ((double)((Ww / c + 31) / 32) + 2.0);
    if (cost < best - 1e-9) { best = cost; wk = c; }
  }
  ResidentParams& p = out->p;
  p = ResidentParams{};
  p.N = N; p.K = K; p.M = M; p.wk = wk;
  p.pieces = nblk < 4 ? nblk : 4;
  p.x_off = kResHead;
  p.lut_off = p.x_off + al128((uint64_t)Mpad * K);
  p.acc_off = p.lut_off + (fmt == kResTL2 ? al128((uint64_t)K * 16) : 0u);
  p.w_off = p.acc_off + (wk > 1 ? al128((uint64_t)nblk * 4 * kResMaxTok * 4) : 0u);
  const uint64_t total = (uint64_t)p.w_off + al128((uint64_t)nblk * 4 * Rb);
  if (total > res_smem_max(fmt)) return false;
  out->grid = grid;
  out->smem = (uint32_t)total;
  return true;
}

template <int FMT, int MT, int MM>
static cudaError_t launch_resident_t(const ResidentPlan& pl, cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attr_once(configured, resident_kernel<FMT, MT, MM>,
                                     (int)res_smem_max(FMT), cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid);
  cfg.blockDim = dim3(kResThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, resident_kernel<FMT, MT, MM>, pl.p);
}

}  // namespace bitnet

using namespace bitnet;

// The resident kernel runs 16 warps per CTA, two CTAs per SM, so the next
// layer's CTA loads its weights while this one computes (one CTA of 32 warps
// per SM measured slower: 6.0 vs 3.4 us per 2B layer).  The products are
// dp4a items: warp-level int8 MMA items (16-row tiles) measured slower here,
// 4.27 vs 2.94 us per 2B layer at one token and 6.36 vs 5.39 at two.

// Whether the resident kernel serves this shape in format fmt (0: I2_S
// ternary, 1: sign bits, 2: I2_S through pair tables).
bool bitnet_resident_fits(int fmt, int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M > 8 || N > 0x7fffffff || K > 0x7fffffff) return false;
  ResidentPlan pl;
  return plan_resident(fmt, (int)M, (int)N, (int)K, num_sms, &pl);
}

bitnet_status bitnet_resident_launch(int fmt, const uint8_t* w, const float* gamma, int N, int K,
                                     const uint16_t* x, int M, uint16_t* y, float* y_f32,
                                     int32_t* acc, int num_sms, cudaStream_t stream) {
  ResidentPlan pl;
  if (!plan_resident(fmt, M, N, K, num_sms, &pl)) return BITNET_ERR_UNSUPPORTED;
  pl.p.w = w; pl.p.gamma = gamma; pl.p.x = x; pl.p.y = y; pl.p.y_f32 = y_f32; pl.p.acc = acc;
  cudaError_t e;
  if (fmt == kResA48) {
    return BITNET_ERR_UNSUPPORTED;             // bitnet_resident_a48_launch
  } else if (fmt == kResTL2) {
    e = launch_resident_t<kResTL2, 1, 1>(pl, stream);
  } else if (fmt == kResW1) {
    if (M == 1) e = launch_resident_t<kResW1, 1, 1>(pl, stream);
    else if (M == 2) e = launch_resident_t<kResW1, 2, 2>(pl, stream);
    else e = launch_resident_t<kResW1, 2, 4>(pl, stream);
  } else {
    if (M == 1) e = launch_resident_t<kResI2S, 1, 1>(pl, stream);
    else if (M == 2) e = launch_resident_t<kResI2S, 2, 2>(pl, stream);
    else e = launch_resident_t<kResI2S, 2, 4>(pl, stream);
  }
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

// One token of BitNet a4.8 on the resident kernel: either rows = the token's
// two code rows [2][K] in the kernel order (q4 then q8) with scale/rowsum
// their [2] scales and row sums (bitnet_quant_act_a48's layout), or rows =
// null and the kernel quantises the bf16 token x [K] itself with n_out 8-bit
// values; acc4/acc8 optional.
bool bitnet_resident_a48_fits(int64_t N, int64_t K, int num_sms) {
  return bitnet_resident_fits(kResA48, 2, N, K, num_sms);
}

bitnet_status bitnet_resident_a48_launch(const uint8_t* w, const float* gamma, int N, int K,
                                         const uint16_t* x, int n_out, const int8_t* rows,
                                         const float* scale, const int32_t* rowsum, uint16_t* y,
                                         float* y_f32, int32_t* acc4, int32_t* acc8,
                                         int num_sms, cudaStream_t stream) {
  ResidentPlan pl;
  if (!plan_resident(kResA48, 2, N, K, num_sms, &pl)) return BITNET_ERR_UNSUPPORTED;
  pl.p.w = w; pl.p.gamma = gamma; pl.p.y = y; pl.p.y_f32 = y_f32; pl.p.acc = acc4;
  pl.p.x = x; pl.p.n_out = n_out;
  pl.p.xq_in = rows; pl.p.s_in = scale; pl.p.rs_in = rowsum; pl.p.acc8 = acc8;
  const cudaError_t e = launch_resident_t<kResA48, 2, 2>(pl, stream);
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
