// BitNet a4.8: 4-bit activations with the largest values split off at 8
// bits, on ternary (I2_S) weights.
//
// youngju.dev "BitNet論文分析：1-Bit LLMの時代", section "BitNet a4.8：
// ハイブリッド量子化戦略": the top fraction of the activation values is
// separated and processed at 8 bits, the rest is quantised to 4 bits.  The
// pages give neither the fraction nor the scales; this library takes, per
// token, the n_out values of largest |x| (ties between equal |x| to the
// lower channel index) as the 8-bit part, and quantises each part with its
// own absmax scale:
//   inliers:  s4 = 7 / max(max|x_in|, 1e-5),    q4 = clamp(rint(x s4), -8, 7)
//   outliers: s8 = 127 / max(max|x_out|, 1e-5), q8 = clamp(rint(x s8), -128, 127)
// each zero at the other part's channels.  Then acc4 = q4 . W_q and
// acc8 = q8 . W_q (exact), and y32 = fp32(acc4) (gamma/s4) + fp32(acc8) (gamma/s8).
//
// Kernels: a quantiser with one CTA per token (a two-level radix select of
// the n_out-th largest 15-bit bf16 magnitude, a block scan that ranks the
// values equal to it by channel, block maxima of the two parts, then the
// two code rows); the tensor-core kernel on the 2M rows (q4 of token m at
// row 2m, q8 at row 2m + 1), which writes the exact accumulators; and a
// combine kernel for y.  For one token the resident decode kernel runs the
// same per-token quantisation (a48_quant_token) in every CTA's prologue and
// combines the two rows in its epilogue.
#include "common.cuh"

namespace bitnet {

constexpr int kA48Threads = 512;

// For a finite bf16 value the magnitude order is the order of its bits with
// the sign cleared.
__device__ __forceinline__ uint32_t mag_key(uint32_t bits16) { return bits16 & 0x7fffu; }

// One warp over a histogram of 32 * PER bins (bin b counts keys whose digit
// is b): the highest bin B whose suffix count (keys with digit >= B, plus
// `above_in` keys above all of them) reaches `need`, and the count above B.
// Lane l holds bins [PER l, PER l + PER); a suffix scan over the lanes and
// one ballot find the lane that holds B, which then walks its own bins.
template <int PER>
__device__ __forceinline__ void warp_select_bin(const unsigned* hist, int need, int above_in,
                                                int lane, int& B, int& above) {
  int loc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) loc += (int)hist[PER * lane + i];
  int suf = loc;                       // sum over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  const unsigned ok = __ballot_sync(0xffffffffu, above_in + suf >= need);
  // lanes 0..L satisfy it (suffix counts do not increase with the lane)
  const int L = ok ? 31 - __clz(ok) : 0;
  const int suf_above = __shfl_sync(0xffffffffu, suf - loc, L);   // lanes > L
  if (lane == L) {
    int acc = above_in + suf_above, b = PER * L;
    for (int i = PER - 1; i >= 0; --i) {
      if (acc + (int)hist[PER * L + i] >= need) { b = PER * L + i; break; }
      acc += (int)hist[PER * L + i];
    }
    B = b;
    above = acc;
  }
  B = __shfl_sync(0xffffffffu, B, L);
  above = __shfl_sync(0xffffffffu, above, L);
}

// One token's a4.8 codes, computed by a block of kA48Threads threads (every
// thread of the block calls it).  Writes, where given (global or shared
// memory): row4 / row8 [K] in the kernels' K order, q4n / q8n [K] in natural
// order; returns the scales and row sums to every thread.
struct A48Token {
  float s4, s8;
  int rs4, rs8;
};

__device__ A48Token a48_quant_token(const uint16_t* __restrict__ xr, int K, int n_out,
                                    int8_t* row4, int8_t* row8, int8_t* q4n, int8_t* q8n) {
  __shared__ unsigned hist[256];
  __shared__ unsigned wsum[kA48Threads / 32];
  __shared__ float wmax4[kA48Threads / 32], wmax8[kA48Threads / 32];
  __shared__ int wrs4[kA48Threads / 32], wrs8[kA48Threads / 32];
  __shared__ int sel[4];        // B, J (threshold key), r (ties taken), flag
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int npiece = K >> 3;                               // 8-value pieces
  const int cp = (npiece + kA48Threads - 1) / kA48Threads;  // pieces per thread
  const int p0 = min(npiece, tid * cp), p1 = min(npiece, p0 + cp);
  auto load8 = [&](int pc, uint32_t (&k)[8], uint32_t (&b)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + pc * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      b[2 * i] = w[i] & 0xffffu;
      b[2 * i + 1] = w[i] >> 16;
      k[2 * i] = mag_key(b[2 * i]);
      k[2 * i + 1] = mag_key(b[2 * i + 1]);
    }
  };

  // ---- select the threshold key T and how many values equal to it are taken
  int T = 0x8000, r = 0;        // n_out == 0: nothing is an outlier
  if (n_out > 0) {
    // level 1: the high 8 bits of the key
    for (int i = tid; i < 256; i += kA48Threads) hist[i] = 0;
    __syncthreads();
    for (int pc = p0; pc < p1; ++pc) {
      uint32_t k[8], b[8];
      load8(pc, k, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) atomicAdd(&hist[k[i] >> 7], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      int B = 0, above = 0;
      warp_select_bin<8>(hist, n_out, 0, lane, B, above);
      if (lane == 0) {
        sel[0] = B;
        sel[1] = above;
      }
    }
    __syncthreads();
    const int B = sel[0];
    int above = sel[1];
    // level 2: the low 7 bits, among keys whose high bits are B
    for (int i = tid; i < 256; i += kA48Threads) hist[i] = 0;
    __syncthreads();
    for (int pc = p0; pc < p1; ++pc) {
      uint32_t k[8], b[8];
      load8(pc, k, b);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((int)(k[i] >> 7) == B) atomicAdd(&hist[k[i] & 127u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      int J = 0, ab = 0;
      warp_select_bin<4>(hist, n_out, above, lane, J, ab);
      if (lane == 0) {
        sel[2] = (B << 7) | J;
        sel[3] = n_out - ab;    // values equal to T taken, in channel order
      }
    }
    __syncthreads();
    T = sel[2];
    r = sel[3];
  }

  // ---- rank the values equal to T by channel (a block scan of per-thread
  // counts over contiguous chunks), classify, and take both parts' maxima
  int ties = 0;
  if (n_out > 0) {
    for (int pc = p0; pc < p1; ++pc) {
      uint32_t k[8], b[8];
      load8(pc, k, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) ties += (int)k[i] == T;
    }
  }
  // exclusive scan of `ties` over the block
  int incl = ties;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = (unsigned)incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += (int)wsum[w];
  int rank = wbase + incl - ties;   // ties before this thread's chunk
  uint32_t a4 = 0, a8 = 0;          // maxima as keys
  for (int pc = p0; pc < p1; ++pc) {
    uint32_t k[8], b[8];
    load8(pc, k, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bool out = (int)k[i] > T;
      if ((int)k[i] == T) { out = rank < r; ++rank; }
      if (out) a8 = max(a8, k[i]);
      else a4 = max(a4, k[i]);
    }
  }
  a4 = __reduce_max_sync(0xffffffffu, a4);
  a8 = __reduce_max_sync(0xffffffffu, a8);
  if (lane == 0) {
    wmax4[warp] = __uint_as_float(a4 << 16);
    wmax8[warp] = __uint_as_float(a8 << 16);
  }
  __syncthreads();
  float m4 = 0.f, m8 = 0.f;
  for (int w = 0; w < kA48Threads / 32; ++w) {
    m4 = fmaxf(m4, wmax4[w]);
    m8 = fmaxf(m8, wmax8[w]);
  }
  const float s4 = __fdiv_rn(7.0f, fmaxf(m4, 1e-5f));
  const float s8 = qscale(m8);

  // ---- quantise both parts (the tie ranks are recomputed in the same order)
  rank = wbase + incl - ties;
  int rs4 = 0, rs8 = 0;
  for (int pc = p0; pc < p1; ++pc) {
    uint32_t k[8], b[8];
    load8(pc, k, b);
    int q4[8], q8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bool out = (int)k[i] > T;
      if ((int)k[i] == T) { out = rank < r; ++rank; }
      const float v = __uint_as_float(b[i] << 16);
      int c4 = __float2int_rn(__fmul_rn(v, s4));
      c4 = c4 < -8 ? -8 : (c4 > 7 ? 7 : c4);
      q4[i] = out ? 0 : c4;
      q8[i] = out ? quant_code_sat(v, s8) : 0;
      rs4 += q4[i];
      rs8 += q8[i];
    }
    const int k0 = pc * 8;
    if (q4n) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        q4n[k0 + i] = (int8_t)q4[i];
        q8n[k0 + i] = (int8_t)q8[i];
      }
    }
    if (row4) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t kk = perm_k(k0 + i);
        row4[kk] = (int8_t)q4[i];
        row8[kk] = (int8_t)q8[i];
      }
    }
  }
  rs4 = __reduce_add_sync(0xffffffffu, rs4);
  rs8 = __reduce_add_sync(0xffffffffu, rs8);
  if (lane == 0) {
    wrs4[warp] = rs4;
    wrs8[warp] = rs8;
  }
  __syncthreads();
  A48Token t{s4, s8, 0, 0};
  for (int w = 0; w < kA48Threads / 32; ++w) {
    t.rs4 += wrs4[w];
    t.rs8 += wrs8[w];
  }
  __syncthreads();                     // the block's shared scratch is free again
  return t;
}

// Quantise one token per CTA.  Outputs (any may be null except the scales):
//   rows   [2M, K] int8 in the kernels' K order (row 2m: q4, row 2m+1: q8)
//   scale  [2M] fp32 (s4, s8), rowsum [2M] int32
//   q4n, q8n [M, K] int8 natural order (for the standalone quantiser)
//   s4, s8 [M] fp32
//   zero   [zero16] 16-byte words cleared after the dependency wait (the
//          split-K scratch of the GEMM that follows), or null
__global__ void __launch_bounds__(kA48Threads) a48_quant_kernel(
    const uint16_t* __restrict__ x, int K, int n_out, int8_t* rows, float* scale, int32_t* rowsum,
    int8_t* q4n, int8_t* q8n, float* s4o, float* s8o, uint4* zero, int64_t zero16) {
  pdl_wait();
  // the consumer of the code rows reads them only after its dependency wait
  pdl_launch_dependents();
  if (zero) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < zero16; i += stride)
      zero[i] = make_uint4(0, 0, 0, 0);
  }
  const int m = blockIdx.x;
  const A48Token t = a48_quant_token(
      x + (int64_t)m * K, K, n_out, rows ? rows + (int64_t)(2 * m) * K : nullptr,
      rows ? rows + (int64_t)(2 * m + 1) * K : nullptr, q4n ? q4n + (int64_t)m * K : nullptr,
      q8n ? q8n + (int64_t)m * K : nullptr);
  if (threadIdx.x == 0) {
    if (scale) {
      scale[2 * m] = t.s4;
      scale[2 * m + 1] = t.s8;
    }
    if (rowsum) {
      rowsum[2 * m] = t.rs4;
      rowsum[2 * m + 1] = t.rs8;
    }
    if (s4o) s4o[m] = t.s4;
    if (s8o) s8o[m] = t.s8;
  }
}

// y32 = fp32(acc4) (gamma / s4) + fp32(acc8) (gamma / s8), from the exact
// accumulators of rows 2m and 2m + 1.
__global__ void __launch_bounds__(256) a48_combine_kernel(
    const int32_t* __restrict__ acc2, const float* __restrict__ scale, const float* gamma, int M,
    int N, uint16_t* y, float* y_f32, int32_t* acc4, int32_t* acc8) {
  pdl_wait();
  const float g = *gamma;
  const int64_t total = (int64_t)M * N;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(o / N), n = (int)(o - (int64_t)m * N);
    const int a4 = acc2[(int64_t)(2 * m) * N + n], a8 = acc2[(int64_t)(2 * m + 1) * N + n];
    const float d4 = __fdiv_rn(g, scale[2 * m]), d8 = __fdiv_rn(g, scale[2 * m + 1]);
    const float y32 = __fadd_rn(__fmul_rn(__int2float_rn(a4), d4), __fmul_rn(__int2float_rn(a8), d8));
    y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
    if (y_f32) y_f32[o] = y32;
    if (acc4) acc4[o] = a4;
    if (acc8) acc8[o] = a8;
  }
}

}  // namespace bitnet

using namespace bitnet;

bitnet_status bitnet_a48_quant_launch(const uint16_t* x, int64_t M, int64_t K, int64_t n_out,
                                      int8_t* rows, float* scale, int32_t* rowsum, int8_t* q4n,
                                      int8_t* q8n, float* s4, float* s8, cudaStream_t stream,
                                      void* zero = nullptr, size_t zero_bytes = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)M);
  cfg.blockDim = dim3(kA48Threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, a48_quant_kernel, x, (int)K, (int)n_out, rows, scale, rowsum, q4n,
                         q8n, s4, s8, static_cast<uint4*>(zero), (int64_t)(zero_bytes / 16));
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_a48_combine_launch(const int32_t* acc2, const float* scale,
                                        const float* gamma, int64_t M, int64_t N, uint16_t* y,
                                        float* y_f32, int32_t* acc4, int32_t* acc8, int num_sms,
                                        cudaStream_t stream) {
  int64_t blocks = (M * N + 255) / 256;
  if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
  a48_combine_kernel<<<(unsigned)blocks, 256, 0, stream>>>(acc2, scale, gamma, (int)M, (int)N, y,
                                                           y_f32, acc4, acc8);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
