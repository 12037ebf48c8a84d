// Per-token absmax int8 activation quantisation (one CTA per token).
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
};

template <bool kF32, bool kPerm>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantArgs a) {
  __shared__ float red_f[8];
  __shared__ int red_i[8];
  __shared__ double red_d[8];
  const int64_t m = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t K = a.K;
  pdl_wait();
  // pass 1: absmax of src*gain (and the sum of squares of src)
  float amax = 0.f;
  double ss = 0.0;
  for (int64_t k = (int64_t)tid * 4; k < K; k += 256 * 4) {
    float v[4];
    if (kF32) {
      const float4 t = *reinterpret_cast<const float4*>(
          static_cast<const float*>(a.src) + m * K + k);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      const uint2 t = *reinterpret_cast<const uint2*>(
          static_cast<const uint16_t*>(a.src) + m * K + k);
      v[0] = __uint_as_float(t.x << 16);
      v[1] = __uint_as_float(t.x & 0xffff0000u);
      v[2] = __uint_as_float(t.y << 16);
      v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (a.sumsq) ss += (double)v[c] * (double)v[c];
      const float g = a.gain ? __fmul_rn(v[c], a.gain[k + c]) : v[c];
      amax = fmaxf(amax, fabsf(g));
    }
  }
  amax = warp_max(amax);
  if (a.sumsq) ss = warp_sum_d(ss);
  if (lane == 0) { red_f[warp] = amax; red_d[warp] = ss; }
  __syncthreads();
  if (tid < 32) {
    float v = lane < 8 ? red_f[lane] : 0.f;
    v = warp_max(v);
    double d = lane < 8 ? red_d[lane] : 0.0;
    if (a.sumsq) d = warp_sum_d(d);
    if (lane == 0) { red_f[0] = v; red_d[0] = d; }
  }
  __syncthreads();
  const float s = qscale(red_f[0]);
  // pass 2: quantise (re-reading the row, now in L1/L2)
  int rs = 0;
  const int64_t step = kPerm ? 16 : 4;
  for (int64_t k = (int64_t)tid * step; k < K; k += 256 * step) {
    int q[16];
#pragma unroll
    for (int c4 = 0; c4 < (kPerm ? 4 : 1); ++c4) {
      const int64_t kk = k + 4 * c4;
      float v[4];
      if (kF32) {
        const float4 t = *reinterpret_cast<const float4*>(
            static_cast<const float*>(a.src) + m * K + kk);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
      } else {
        const uint2 t = *reinterpret_cast<const uint2*>(
            static_cast<const uint16_t*>(a.src) + m * K + kk);
        v[0] = __uint_as_float(t.x << 16);
        v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16);
        v[3] = __uint_as_float(t.y & 0xffff0000u);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float g = a.gain ? __fmul_rn(v[c], a.gain[kk + c]) : v[c];
        q[4 * c4 + c] = quant_code(g, s);
        rs += q[4 * c4 + c];
      }
    }
    if (kPerm) {
      // slot 4*t + b holds natural index 4*b + t
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        w[t] = (uint32_t)(q[t] & 0xff) | ((uint32_t)(q[4 + t] & 0xff) << 8) |
               ((uint32_t)(q[8 + t] & 0xff) << 16) | ((uint32_t)(q[12 + t] & 0xff) << 24);
      *reinterpret_cast<uint4*>(a.xq + m * a.ld_q + k) = make_uint4(w[0], w[1], w[2], w[3]);
      if (a.xq_natural) {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t n = (uint32_t)(q[4 * c4] & 0xff) | ((uint32_t)(q[4 * c4 + 1] & 0xff) << 8) |
                             ((uint32_t)(q[4 * c4 + 2] & 0xff) << 16) |
                             ((uint32_t)(q[4 * c4 + 3] & 0xff) << 24);
          *reinterpret_cast<uint32_t*>(a.xq_natural + m * K + k + 4 * c4) = n;
        }
      }
    } else {
      const uint32_t n = (uint32_t)(q[0] & 0xff) | ((uint32_t)(q[1] & 0xff) << 8) |
                         ((uint32_t)(q[2] & 0xff) << 16) | ((uint32_t)(q[3] & 0xff) << 24);
      *reinterpret_cast<uint32_t*>(a.xq + m * a.ld_q + k) = n;
    }
  }
  rs = warp_sum_i(rs);
  if (lane == 0) red_i[warp] = rs;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < 8; ++w) t += red_i[w];
    a.scale[m] = s;
    if (a.rowsum) a.rowsum[m] = t;
    if (a.sumsq) a.sumsq[m] = red_d[0];
  }
  pdl_launch_dependents();
}

}  // namespace bitnet

using namespace bitnet;

// Launch helper used by the C ABI (kF32 / kPerm chosen at runtime).
bitnet_status bitnet_quant_launch(const void* src, bool src_f32, const float* gain, int64_t M,
                                  int64_t K, int8_t* xq, int64_t ld_q, bool perm, float* scale,
                                  int32_t* rowsum, double* sumsq, int8_t* xq_natural,
                                  cudaStream_t stream) {
  QuantArgs a{src, gain, M, K, xq, ld_q, scale, rowsum, sumsq, xq_natural};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)M);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (src_f32) {
    e = perm ? cudaLaunchKernelEx(&cfg, quant_rows_kernel<true, true>, a)
             : cudaLaunchKernelEx(&cfg, quant_rows_kernel<true, false>, a);
  } else {
    e = perm ? cudaLaunchKernelEx(&cfg, quant_rows_kernel<false, true>, a)
             : cudaLaunchKernelEx(&cfg, quant_rows_kernel<false, false>, a);
  }
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
