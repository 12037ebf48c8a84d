// Per-token absmax int8 activation quantisation: one warp per token for many
// short rows, one 256-thread CTA per token for few tokens or long rows.
//
// youngju.dev "BitNet論文分析：1-Bit LLMの時代", section "Absmean量子化関数",
// BitLinear_b158.activation_quant: per-token absmax scale, round, clamp.
// s = 127 / max(max|v|, 1e-5); q = clamp(rint(v * s), -128, 127), v = src * gain.
//
// Source is bf16 bits or fp32 (the FFN's h'); the optional gain is the RMSNorm
// weight (the per-token RMS factor itself is folded into the dequant scale).
// The output is either the natural [M,K] layout or the kernels' permuted
// layout (perm_k) that lines activation words up with the packed code planes.
#include "common.cuh"

namespace bitnet {

struct QuantArgs {
  const void* src;        // [M,K] bf16 bits or fp32
  const float* gain;      // [K] or null
  int64_t M, K;
  int8_t* xq;             // [M, ld_q] written
  int64_t ld_q;           // row stride of xq in bytes (>= K)
  float* scale;           // [M] written
  int32_t* rowsum;        // [M] or null
  double* sumsq;          // [M] or null: sum over k of src^2 (not the gained value)
  int8_t* xq_natural;     // optional extra natural-layout copy (debug), [M,K]
  const float* amax_in;   // [M] or null: the absmax to quantise with (a tensor-
                          // parallel shard uses the all-reduced one)
  float* amax_out;        // [M] or null: this row's absmax of src * gain
  uint4* zero;            // or null: a scratch range the grid clears after its
  int64_t zero16;         // dependency wait (16-byte words), e.g. the split-K
                          // accumulators of the kernel that follows
};

// Clear the scratch range, grid-stride over the whole launch.
__device__ __forceinline__ void clear_scratch(const QuantArgs& a) {
  if (!a.zero) return;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.zero16; i += stride)
    a.zero[i] = make_uint4(0, 0, 0, 0);
}

// 8 consecutive source values as floats (one 16-byte load of bf16, two of fp32).
template <bool kF32>
__device__ __forceinline__ void load8(const void* src, int64_t idx, float (&v)[8]) {
  if (kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 t = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + idx);
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}
template <bool kF32>
__device__ __forceinline__ void load4(const void* src, int64_t idx, float (&v)[4]) {
  if (kF32) {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + idx);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const uint2 t = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(src) + idx);
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return __byte_perm(__byte_perm((uint32_t)a, (uint32_t)b, 0x0040),
                     __byte_perm((uint32_t)c, (uint32_t)d, 0x0040), 0x5410);
}

// One warp per token: two passes over the row (the second mostly from L1),
// reductions by shuffles only.  kPerm needs K % 16 == 0.
template <bool kF32, bool kPerm>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  pdl_wait();
  // the kernel that consumes the codes may start its own set-up (and its
  // weight loads) now; it reads the codes only after its dependency wait
  pdl_launch_dependents();
  clear_scratch(a);
  if (m < a.M) {
    const int64_t K = a.K;
    const int64_t base = m * K;
    // rows start 16-byte aligned only when K % 8 == 0 (bf16) ; otherwise use
    // 4-element chunks (8-byte bf16 loads, 4-byte code stores) throughout
    const bool v8 = (K & 7) == 0;
    const int64_t K8 = v8 ? K : 0;
    // pass 1: absmax of src * gain, sum of squares of src
    float amax = 0.f;
    double ss = 0.0;
#pragma unroll 4
    for (int64_t k = (int64_t)lane * 8; k < K8; k += 256) {
      float v[8];
      load8<kF32>(a.src, base + k, v);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (a.sumsq) ss += (double)v[c] * (double)v[c];
        const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
        amax = fmaxf(amax, fabsf(g));
      }
    }
    for (int64_t k = K8 + (int64_t)lane * 4; k < K; k += 128) {
      float v[4];
      load4<kF32>(a.src, base + k, v);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (a.sumsq) ss += (double)v[c] * (double)v[c];
        const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
        amax = fmaxf(amax, fabsf(g));
      }
    }
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (a.sumsq) ss = warp_sum_d(ss);
    if (a.amax_out && lane == 0) a.amax_out[m] = amax;
    const float s = qscale(a.amax_in ? a.amax_in[m] : amax);
    // pass 2: quantise
    int rs = 0;
    if (kPerm) {
      for (int64_t k = (int64_t)lane * 16; k < K; k += 512) {
        float v0[8], v1[8];
        load8<kF32>(a.src, base + k, v0);
        load8<kF32>(a.src, base + k + 8, v1);
        int q[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float g0 = a.gain ? __fmul_rn(v0[c], a.gain[k + c]) : v0[c];
          const float g1 = a.gain ? __fmul_rn(v1[c], a.gain[k + 8 + c]) : v1[c];
          q[c] = quant_code_sat(g0, s);
          q[8 + c] = quant_code_sat(g1, s);
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) rs += q[c];
        // slot 4*t + b holds natural index 4*b + t
        *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + k) =
            make_uint4(pack4(q[0], q[4], q[8], q[12]), pack4(q[1], q[5], q[9], q[13]),
                       pack4(q[2], q[6], q[10], q[14]), pack4(q[3], q[7], q[11], q[15]));
        if (a.xq_natural)
          *reinterpret_cast<uint4*>(a.xq_natural + m * K + k) =
              make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                         pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
      }
    } else {
#pragma unroll 4
      for (int64_t k = (int64_t)lane * 8; k < K8; k += 256) {
        float v[8];
        load8<kF32>(a.src, base + k, v);
        int q[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
          q[c] = quant_code_sat(g, s);
          rs += q[c];
        }
        *reinterpret_cast<uint2*>(a.xq + m * a.ld_q + k) =
            make_uint2(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]));
      }
      for (int64_t k = K8 + (int64_t)lane * 4; k < K; k += 128) {
        float v[4];
        load4<kF32>(a.src, base + k, v);
        int q[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
          q[c] = quant_code_sat(g, s);
          rs += q[c];
        }
        *reinterpret_cast<uint32_t*>(a.xq + m * a.ld_q + k) = pack4(q[0], q[1], q[2], q[3]);
      }
    }
    rs = __reduce_add_sync(0xffffffffu, rs);
    if (lane == 0) {
      a.scale[m] = s;
      if (a.rowsum) a.rowsum[m] = rs;
      if (a.sumsq) a.sumsq[m] = ss;
    }
  }
}

// One 256-thread CTA per token, block reductions through shared memory: for
// few tokens (a warp per token would leave almost the whole GPU idle) and
// for long rows (a warp per token is a long chain of dependent loads).  Same
// arithmetic as quant_rows_kernel: absmax and the integer row sum do not
// depend on order; the fp64 sum of squares (the FFN's RMS factor) may differ
// in rounding order only.
template <bool kF32, bool kPerm>
__global__ void __launch_bounds__(256) quant_token_kernel(QuantArgs a) {
  __shared__ float s_max[8];
  __shared__ double s_ss[8];
  __shared__ int s_rs[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t m = blockIdx.x;
  const int64_t K = a.K;
  const int64_t base = m * K;
  pdl_wait();
  pdl_launch_dependents();
  clear_scratch(a);
  // pass 1: absmax of src * gain, sum of squares of src; groups of 8
  // (16-byte bf16 loads) when rows start 16-byte aligned, else of 4
  float amax = 0.f;
  double ss = 0.0;
  const int64_t K8 = (K & 7) == 0 ? K : 0;
#pragma unroll 2
  for (int64_t k = (int64_t)threadIdx.x * 8; k < K8; k += 2048) {
    float v[8];
    load8<kF32>(a.src, base + k, v);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (a.sumsq) ss += (double)v[c] * (double)v[c];
      const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
      amax = fmaxf(amax, fabsf(g));
    }
  }
  for (int64_t k = K8 + (int64_t)threadIdx.x * 4; k < K; k += 1024) {
    float v[4];
    load4<kF32>(a.src, base + k, v);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (a.sumsq) ss += (double)v[c] * (double)v[c];
      const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
      amax = fmaxf(amax, fabsf(g));
    }
  }
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  if (a.sumsq) ss = warp_sum_d(ss);
  if (lane == 0) {
    s_max[warp] = amax;
    s_ss[warp] = ss;
  }
  __syncthreads();
  float am = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) am = fmaxf(am, s_max[w]);
  if (a.amax_out && threadIdx.x == 0) a.amax_out[m] = am;
  const float s = qscale(a.amax_in ? a.amax_in[m] : am);
  // pass 2: quantise (groups of 16 for the permuted layout, else 4)
  int rs = 0;
  if (kPerm) {
    for (int64_t k = (int64_t)threadIdx.x * 16; k < K; k += 4096) {
      float v0[8], v1[8];
      load8<kF32>(a.src, base + k, v0);
      load8<kF32>(a.src, base + k + 8, v1);
      int q[16];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float g0 = a.gain ? __fmul_rn(v0[c], a.gain[k + c]) : v0[c];
        const float g1 = a.gain ? __fmul_rn(v1[c], a.gain[k + 8 + c]) : v1[c];
        q[c] = quant_code_sat(g0, s);
        q[8 + c] = quant_code_sat(g1, s);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) rs += q[c];
      // slot 4*t + b holds natural index 4*b + t
      *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + k) =
          make_uint4(pack4(q[0], q[4], q[8], q[12]), pack4(q[1], q[5], q[9], q[13]),
                     pack4(q[2], q[6], q[10], q[14]), pack4(q[3], q[7], q[11], q[15]));
      if (a.xq_natural)
        *reinterpret_cast<uint4*>(a.xq_natural + m * K + k) =
            make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                       pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
    }
  } else {
    for (int64_t k = (int64_t)threadIdx.x * 4; k < K; k += 1024) {
      float v[4];
      load4<kF32>(a.src, base + k, v);
      int q[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
        q[c] = quant_code_sat(g, s);
        rs += q[c];
      }
      *reinterpret_cast<uint32_t*>(a.xq + m * a.ld_q + k) = pack4(q[0], q[1], q[2], q[3]);
    }
  }
  rs = __reduce_add_sync(0xffffffffu, rs);
  if (lane == 0) s_rs[warp] = rs;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    double d = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      t += s_rs[w];
      d += s_ss[w];
    }
    a.scale[m] = s;
    if (a.rowsum) a.rowsum[m] = t;
    if (a.sumsq) a.sumsq[m] = d;
  }
}

// quant_token_kernel for bf16 rows of at most 8192 values with K % 16 == 0:
// each thread loads its (at most two) 16-value groups once and keeps them in
// registers for the second pass, so a token costs one round of loads instead
// of two.  Same arithmetic and outputs as quant_token_kernel.
template <bool kPerm>
__global__ void __launch_bounds__(256) quant_token_cached_kernel(QuantArgs a) {
  constexpr int kGroups = 2;
  __shared__ float s_max[8];
  __shared__ double s_ss[8];
  __shared__ int s_rs[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t m = blockIdx.x;
  const int64_t K = a.K;
  const uint16_t* row = static_cast<const uint16_t*>(a.src) + m * K;
  pdl_wait();
  pdl_launch_dependents();
  clear_scratch(a);
  uint4 v[kGroups][2];
#pragma unroll
  for (int i = 0; i < kGroups; ++i) {
    const int64_t k = ((int64_t)threadIdx.x + 256 * i) * 16;
    v[i][0] = v[i][1] = make_uint4(0, 0, 0, 0);
    if (k < K) {
      v[i][0] = *reinterpret_cast<const uint4*>(row + k);
      v[i][1] = *reinterpret_cast<const uint4*>(row + k + 8);
    }
  }
  auto value = [&](int i, int c) {             // value c of group i, as fp32
    const uint4& h = v[i][c >> 3];
    const int j = (c & 7) >> 1;
    const uint32_t w = j == 0 ? h.x : j == 1 ? h.y : j == 2 ? h.z : h.w;
    return __uint_as_float((c & 1) ? (w & 0xffff0000u) : (w << 16));
  };
  float amax = 0.f;
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < kGroups; ++i) {
    const int64_t k = ((int64_t)threadIdx.x + 256 * i) * 16;
    if (k < K) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float x = value(i, c);
        if (a.sumsq) ss += (double)x * (double)x;
        const float g = a.gain ? __fmul_rn(x, a.gain[k + c]) : x;
        amax = fmaxf(amax, fabsf(g));
      }
    }
  }
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  if (a.sumsq) ss = warp_sum_d(ss);
  if (lane == 0) {
    s_max[warp] = amax;
    s_ss[warp] = ss;
  }
  __syncthreads();
  float am = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) am = fmaxf(am, s_max[w]);
  if (a.amax_out && threadIdx.x == 0) a.amax_out[m] = am;
  const float s = qscale(a.amax_in ? a.amax_in[m] : am);
  int rs = 0;
#pragma unroll
  for (int i = 0; i < kGroups; ++i) {
    const int64_t k = ((int64_t)threadIdx.x + 256 * i) * 16;
    if (k < K) {
      int q[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float x = value(i, c);
        q[c] = quant_code_sat(a.gain ? __fmul_rn(x, a.gain[k + c]) : x, s);
        rs += q[c];
      }
      const uint4 nat = make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                                   pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
      if (kPerm) {
        // slot 4*t + b holds natural index 4*b + t
        *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + k) =
            make_uint4(pack4(q[0], q[4], q[8], q[12]), pack4(q[1], q[5], q[9], q[13]),
                       pack4(q[2], q[6], q[10], q[14]), pack4(q[3], q[7], q[11], q[15]));
        if (a.xq_natural) *reinterpret_cast<uint4*>(a.xq_natural + m * K + k) = nat;
      } else {
        *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + k) = nat;
      }
    }
  }
  rs = __reduce_add_sync(0xffffffffu, rs);
  if (lane == 0) s_rs[warp] = rs;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    double d = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      t += s_rs[w];
      d += s_ss[w];
    }
    a.scale[m] = s;
    if (a.rowsum) a.rowsum[m] = t;
    if (a.sumsq) a.sumsq[m] = d;
  }
}

// Plain per-token quantiser for the tensor-core path (bf16 rows, no gain, no
// norm statistics, K % 16 == 0, K <= 8192).  A CTA is one token's team (K/32
// threads rounded up to whole warps, two groups of 16 values per thread) and
// loops over the tokens blockIdx.x, + gridDim.x, ...  Thread 0 keeps the
// row of the CTA's next token on its way into a two-stage shared-memory ring
// (bulk copies, completion on the stage's mbarrier) while the team reduces
// and quantises the current one, so each SM always has rows in flight.  Two
// stages rather than more: the ring's size sets how many CTAs fit on an SM,
// and more resident teams measured faster than deeper rings (prefill down
// input: 16.8 us with two stages, 18.9 us with four).  Same arithmetic and
// outputs as quant_token_cached_kernel.
constexpr int kQStages = 2;

template <bool kPerm>
__global__ void __launch_bounds__(256) quant_stream_kernel(QuantArgs a) {
  extern __shared__ __align__(16) uint8_t q_smem[];
  __shared__ uint64_t full[kQStages];
  __shared__ float s_max[8];
  __shared__ int s_rs[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int64_t K = a.K;
  const uint32_t row_bytes = (uint32_t)K * 2;
  const int64_t kg[2] = {(int64_t)tid * 16, ((int64_t)tid + blockDim.x) * 16};
  const bool on[2] = {kg[0] < K, kg[1] < K};
  const uint16_t* src = static_cast<const uint16_t*>(a.src);
  const int64_t step = gridDim.x;
  const uint64_t pol = policy_evict_first();
  if (tid == 0) {
    for (int i = 0; i < kQStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  auto issue = [&](int64_t m, int st) {        // thread 0: row m into stage st
    uint8_t* dst = q_smem + (size_t)st * row_bytes;
    const uint8_t* g = reinterpret_cast<const uint8_t*>(src + m * K);
    mbar_arrive_expect_tx(&full[st], row_bytes);
    for (uint32_t off = 0; off < row_bytes; off += 4096u) {
      const uint32_t nb = row_bytes - off < 4096u ? row_bytes - off : 4096u;
      bulk_g2s(dst + off, g + off, nb, &full[st], pol);
    }
  };
  if (tid == 0)
    for (int i = 0; i < kQStages; ++i)
      if (blockIdx.x + i * step < a.M) issue(blockIdx.x + i * step, i);
  clear_scratch(a);
  int it = 0;
  for (int64_t m = blockIdx.x; m < a.M; m += step, ++it) {
    const int st = it % kQStages;
    bool ok = mbar_wait(&full[st], (uint32_t)(it / kQStages) & 1u);
    const uint16_t* row = reinterpret_cast<const uint16_t*>(q_smem + (size_t)st * row_bytes);
    uint4 cur[2][2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      cur[i][0] = cur[i][1] = make_uint4(0, 0, 0, 0);
      if (on[i]) {
        cur[i][0] = *reinterpret_cast<const uint4*>(row + kg[i]);
        cur[i][1] = *reinterpret_cast<const uint4*>(row + kg[i] + 8);
      }
    }
    auto value = [&](int i, int c) {           // value c of group i, as fp32
      const uint4& h = cur[i][c >> 3];
      const int j = (c & 7) >> 1;
      const uint32_t w = j == 0 ? h.x : j == 1 ? h.y : j == 2 ? h.z : h.w;
      return __uint_as_float((c & 1) ? (w & 0xffff0000u) : (w << 16));
    };
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 16; ++c) amax = fmaxf(amax, fabsf(value(i, c)));   // padding is 0
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0) s_max[warp] = amax;
    // every thread has its values in registers: the stage is free again
    ok = __syncthreads_and(ok) != 0;
    if (!ok) {
      // a row copy did not complete in time (recorded): wait, bounded, for
      // the copies still in flight into this CTA's ring, then stop
      if (tid == 0)
        for (int i = 0; i < kQStages; ++i)
          if (m + i * step < a.M) (void)mbar_wait(&full[(it + i) % kQStages], (uint32_t)((it + i) / kQStages) & 1u);
      return;
    }
    if (tid == 0 && m + kQStages * step < a.M) issue(m + kQStages * step, st);
    float am = s_max[0];
    for (int w = 1; w < nw; ++w) am = fmaxf(am, s_max[w]);
    const float s = qscale(am);
    uint32_t rs = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (on[i]) {
        int q[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) q[c] = quant_code_sat(value(i, c), s);
        uint4 o;
        if (kPerm)   // slot 4*t + b holds natural index 4*b + t
          o = make_uint4(pack4(q[0], q[4], q[8], q[12]), pack4(q[1], q[5], q[9], q[13]),
                         pack4(q[2], q[6], q[10], q[14]), pack4(q[3], q[7], q[11], q[15]));
        else
          o = make_uint4(pack4(q[0], q[1], q[2], q[3]), pack4(q[4], q[5], q[6], q[7]),
                         pack4(q[8], q[9], q[10], q[11]), pack4(q[12], q[13], q[14], q[15]));
        *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + kg[i]) = o;
        // the row sum from the packed codes (signed bytes times 1)
        rs = (uint32_t)__dp4a((int)o.x, 0x01010101, (int)rs);
        rs = (uint32_t)__dp4a((int)o.y, 0x01010101, (int)rs);
        rs = (uint32_t)__dp4a((int)o.z, 0x01010101, (int)rs);
        rs = (uint32_t)__dp4a((int)o.w, 0x01010101, (int)rs);
      }
    }
    const int rw = __reduce_add_sync(0xffffffffu, (int)rs);
    if (lane == 0) s_rs[warp] = rw;
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < nw; ++w) t += s_rs[w];
      a.scale[m] = s;
      if (a.rowsum) a.rowsum[m] = t;
    }
  }
}

}  // namespace bitnet

using namespace bitnet;

// Launch helper used by the C ABI (kF32 / kPerm chosen at runtime).
bitnet_status bitnet_quant_launch(const void* src, bool src_f32, const float* gain, int64_t M,
                                  int64_t K, int8_t* xq, int64_t ld_q, bool perm, float* scale,
                                  int32_t* rowsum, double* sumsq, int8_t* xq_natural,
                                  cudaStream_t stream, const float* amax_in = nullptr,
                                  float* amax_out = nullptr, void* zero = nullptr,
                                  size_t zero_bytes = 0) {
  QuantArgs a{src,      gain,     M,
              K,        xq,       ld_q,
              scale,    rowsum,   sumsq,
              xq_natural, amax_in, amax_out,
              static_cast<uint4*>(zero), (int64_t)(zero_bytes / 16)};
  cudaLaunchConfig_t cfg = {};
  // a CTA per token for up to 256 tokens or rows longer than 4096 values;
  // else a warp per token (measured faster for many short rows)
  const bool per_token = M <= 256 || K > 4096;
  cfg.gridDim = dim3((unsigned)(per_token ? M : (M + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  // plain bf16 rows of at most 8192 values in 16-byte-aligned groups of 16
  // (the tensor-core path's quantiser): the persistent streaming kernel, as
  // many token teams as fit on the SMs
  const bool plain = !src_f32 && !gain && !sumsq && !xq_natural && !amax_in && !amax_out &&
                     K % 16 == 0 && K <= 8192 && ld_q % 16 == 0;
  if (plain) {
    const int warps = (int)((K + 1023) / 1024);   // 32 values per thread
    // the ring (kQStages rows of up to 16 KB) may exceed the 48 KB default
    static std::atomic<uint64_t> configured[2];
    e = perm ? set_smem_attr_once(configured[1], quant_stream_kernel<true>, kQStages * 8192 * 2)
             : set_smem_attr_once(configured[0], quant_stream_kernel<false>, kQStages * 8192 * 2);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    // resident CTAs per SM for this row length (ring size), computed once
    static std::atomic<int> occ[2][8192 / 16 + 1];
    std::atomic<int>& o = occ[perm ? 1 : 0][K / 16];
    int per_sm = o.load(std::memory_order_relaxed);
    if (per_sm == 0) {
      const size_t smem = (size_t)kQStages * (size_t)K * 2;
      e = perm ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_stream_kernel<true>,
                                                               32 * warps, smem)
               : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_stream_kernel<false>,
                                                               32 * warps, smem);
      if (e != cudaSuccess || per_sm < 1) per_sm = 1;
      o.store(per_sm, std::memory_order_relaxed);
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BITNET_ERR_CUDA;
    const int64_t slots = (int64_t)sms * per_sm;
    cfg.gridDim = dim3((unsigned)(M < slots ? M : slots));
    cfg.blockDim = dim3(32 * warps);
    cfg.dynamicSmemBytes = (size_t)kQStages * (size_t)K * 2;
    e = perm ? cudaLaunchKernelEx(&cfg, quant_stream_kernel<true>, a)
             : cudaLaunchKernelEx(&cfg, quant_stream_kernel<false>, a);
    return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
  }
  // bf16 rows of at most 8192 values in 16-byte-aligned groups of 16: the
  // register-cached CTA-per-token kernel
  const bool cached = per_token && !src_f32 && K % 16 == 0 && K <= 8192 && ld_q % 16 == 0;
  if (cached) {
    e = perm ? cudaLaunchKernelEx(&cfg, quant_token_cached_kernel<true>, a)
             : cudaLaunchKernelEx(&cfg, quant_token_cached_kernel<false>, a);
  } else if (per_token) {
    if (src_f32) {
      e = perm ? cudaLaunchKernelEx(&cfg, quant_token_kernel<true, true>, a)
               : cudaLaunchKernelEx(&cfg, quant_token_kernel<true, false>, a);
    } else {
      e = perm ? cudaLaunchKernelEx(&cfg, quant_token_kernel<false, true>, a)
               : cudaLaunchKernelEx(&cfg, quant_token_kernel<false, false>, a);
    }
  } else if (src_f32) {
    e = perm ? cudaLaunchKernelEx(&cfg, quant_rows_kernel<true, true>, a)
             : cudaLaunchKernelEx(&cfg, quant_rows_kernel<true, false>, a);
  } else {
    e = perm ? cudaLaunchKernelEx(&cfg, quant_rows_kernel<false, true>, a)
             : cudaLaunchKernelEx(&cfg, quant_rows_kernel<false, false>, a);
  }
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
