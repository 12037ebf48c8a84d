// Absmean ternary quantisation and I2_S 2-bit packing on the GPU.
//
// youngju.dev "BitNet論文分析：1-Bit LLMの時代", section "Absmean量子化関数"
// (gamma = mean|W|, W_q = clamp(round(W / (gamma + 1e-5)), -1, 1)) and section
// "アーキテクチャ概要" (I2_S codes 00 = -1, 01 = 0, 10 = +1).
//
// gamma is the fp32 value nearest to the exact mean of |W|, so it does not
// depend on the order in which thousands of threads add: every |w| is
// m * 2^(e-150) with an integer mantissa m, so the kernels add the mantissas
// exactly into one 64-bit integer per exponent e (bucket), and a one-thread
// kernel turns the 256 buckets into the correctly rounded quotient.
#include "common.cuh"

namespace bitnet {

// Workspace layout of bitnet_pack_weights.
struct PackWs {
  unsigned long long bucket[256];
  unsigned int nonfinite;
  float den;                 // gamma + 1e-5f
};

__global__ void __launch_bounds__(256) gamma_bucket_kernel(const float4* __restrict__ W,
                                                            int64_t n4, PackWs* ws) {
  __shared__ unsigned long long sb[256];
  sb[threadIdx.x] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  bool bad = false;
  // warp-uniform loop: every lane runs the same number of iterations, so the
  // warp-collective match/reduce below always sees the full warp
  for (int64_t base = warp_global * 32; base < n4; base += nwarps * 32) {
    const int64_t i = base + lane;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const bool valid = i < n4;
    if (valid) v = __ldcs(&W[i]);
    float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t bits = __float_as_uint(e4[c]) & 0x7fffffffu;
      uint32_t e = bits >> 23;
      uint32_t m = bits & 0x7fffffu;
      if (e == 255u) { bad = bad || valid; m = 0; }
      if (e != 0u) m |= 0x800000u;
      if (e == 0u) e = 1u;          // subnormals share the grid of e = 1
      if (e == 255u) e = 1u;
      if (!valid) { m = 0; e = 1u; }
      const uint32_t grp = __match_any_sync(0xffffffffu, e);
      const uint32_t sum = __reduce_add_sync(grp, m);   // < 32 * 2^24, exact
      if (lane == __ffs(grp) - 1 && sum != 0u)
        atomicAdd(&sb[e], (unsigned long long)sum);
    }
  }
  if (bad) atomicExch(&ws->nonfinite, 1u);
  __syncthreads();
  const unsigned long long t = sb[threadIdx.x];
  if (t) atomicAdd(&ws->bucket[threadIdx.x], t);
}

// Exact sum I = sum_e bucket[e] * 2^(e-1) (units of 2^-149) as 32-bit limbs.
constexpr int kLimbs = 11;   // 352 bits > 254 + 64

__device__ inline int big_bit(const uint32_t* L, int i) {
  return (i < 0) ? 0 : (L[i >> 5] >> (i & 31)) & 1;
}

__global__ void gamma_finalize_kernel(PackWs* ws, unsigned long long count, float* gamma_out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (ws->nonfinite) {
    *gamma_out = __uint_as_float(0x7fc00000u);
    ws->den = __uint_as_float(0x7fc00000u);
    record_error(BITNET_ERR_NONFINITE);
    return;
  }
  uint32_t L[kLimbs];
  for (int i = 0; i < kLimbs; ++i) L[i] = 0;
  for (int e = 1; e < 255; ++e) {
    unsigned long long v = ws->bucket[e];
    if (!v) continue;
    const int sh = e - 1;
    int limb = sh >> 5, off = sh & 31;
    // add v << off into limbs starting at `limb`, with carry
    unsigned long long lo = (v << off) & 0xffffffffull;
    unsigned long long mid = (off ? (v >> (32 - off)) : (v >> 32)) & 0xffffffffull;
    unsigned long long hi = off ? (v >> (64 - off)) : 0ull;
    unsigned long long parts[3] = {lo, mid, hi};
    unsigned long long carry = 0;
    for (int p = 0; limb + p < kLimbs; ++p) {
      unsigned long long add = (p < 3 ? parts[p] : 0ull) + carry;
      if (p >= 3 && add == 0) break;
      unsigned long long s = (unsigned long long)L[limb + p] + add;
      L[limb + p] = (uint32_t)s;
      carry = s >> 32;
    }
  }
  int top = -1;
  for (int i = kLimbs * 32 - 1; i >= 0; --i)
    if (big_bit(L, i)) { top = i; break; }
  float g;
  if (top < 0) {
    g = 0.0f;
  } else {
    // Long division of I by count, most significant quotient bit first.  The
    // leading quotient bit sits at index p (I/count in [2^p, 2^(p+1))); keep
    // bits p .. max(p-23, 0) (24 bits, or the 2^-149 subnormal grid), then a
    // guard bit and a sticky bit.
    const unsigned long long D = count;
    unsigned long long r = 0;
    int p = -1000000, stop = 0;
    uint32_t mant = 0;
    bool guard = false, sticky = false, found = false;
    for (int idx = top;; --idx) {
      r = (r << 1) | (unsigned long long)big_bit(L, idx);
      uint32_t qb = 0;
      if (r >= D) { r -= D; qb = 1; }
      if (!found) {
        if (!qb) {
          if (idx == -1) break;            // below 2^-150: rounds to zero
          continue;
        }
        found = true;
        p = idx;
        stop = p - 23 > 0 ? p - 23 : 0;
      }
      if (idx >= stop) {
        mant = (mant << 1) | qb;
        continue;
      }
      guard = qb != 0;
      bool low = r != 0;
      for (int k = idx - 1; k >= 0 && !low; --k) low = big_bit(L, k) != 0;
      sticky = low;
      break;
    }
    if (guard && (sticky || (mant & 1u))) ++mant;
    uint32_t bits;
    if (!found) {
      bits = 0u;
    } else if (stop == 0 && p < 23) {
      bits = mant;                         // subnormal (or 2^-126 after carry)
    } else {
      if (mant == (1u << 24)) { mant >>= 1; ++p; }
      const int biased = p - 22;           // (p - 149) + 127
      bits = biased >= 255 ? 0x7f800000u : ((uint32_t)biased << 23) | (mant & 0x7fffffu);
    }
    g = __uint_as_float(bits);
  }
  *gamma_out = g;
  ws->den = __fadd_rn(g, 1e-5f);
}

// One output byte (four weights along K) per thread.
__global__ void __launch_bounds__(256) ternary_pack_kernel(const float4* __restrict__ W,
                                                            int64_t nbytes,
                                                            const PackWs* __restrict__ ws,
                                                            uint8_t* __restrict__ packed) {
  const float den = ws->den;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = __ldcs(&W[i]);
    const float e4[4] = {v.x, v.y, v.z, v.w};
    uint32_t byte = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float t = rintf(__fdiv_rn(e4[c], den));
      t = fminf(fmaxf(t, -1.0f), 1.0f);
      const uint32_t code = (uint32_t)((int)t + 1);
      byte |= code << (2 * c);
    }
    packed[i] = (uint8_t)byte;
  }
}

// BitNet v1 sign weights (youngju.dev page, section "BitNet v1：BitLinearの誕生"
// > "1-Bit重みとSign関数": W_b = +1 where W >= 0, -1 where W < 0): one output
// byte (eight weights along K, bit i for weight 8j + i, 1 for +1) per thread.
__global__ void __launch_bounds__(256) sign_pack_kernel(const float4* __restrict__ W,
                                                         int64_t nbytes,
                                                         uint8_t* __restrict__ packed) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(&W[2 * i]), b = __ldcs(&W[2 * i + 1]);
    const float e8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t byte = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) byte |= (e8[c] >= 0.0f ? 1u : 0u) << c;
    packed[i] = (uint8_t)byte;
  }
}

// Sign bits -> I2_S codes of the same +-1 matrix (a +-1 matrix is a ternary
// one): bit 1 -> code 10 (+1), bit 0 -> code 00 (-1).  One sign byte becomes
// two code bytes.
__global__ void __launch_bounds__(256) sign_to_i2s_kernel(const uint8_t* __restrict__ sign,
                                                           int64_t nbytes,
                                                           uint8_t* __restrict__ codes) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t v = sign[i];
    uint32_t out = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) out |= ((v >> c) & 1u) << (2 * c + 1);
    codes[2 * i] = (uint8_t)(out & 0xffu);
    codes[2 * i + 1] = (uint8_t)(out >> 8);
  }
}

}  // namespace bitnet

using namespace bitnet;

size_t bitnet_pack_workspace_size_impl() { return 4096; }

bitnet_status bitnet_pack_w1_launch(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                    float* alpha, void* workspace, cudaStream_t stream,
                                    int num_sms) {
  PackWs* ws = reinterpret_cast<PackWs*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(PackWs), stream) != cudaSuccess) return BITNET_ERR_CUDA;
  const int64_t total = N * K;
  const int64_t n4 = total / 4;
  int grid = num_sms * 4;
  const int64_t need = (n4 + 255) / 256;
  if (need < grid) grid = (int)(need > 0 ? need : 1);
  // alpha = mean |W|: the same exact mean as gamma
  gamma_bucket_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(W), n4, ws);
  gamma_finalize_kernel<<<1, 32, 0, stream>>>(ws, (unsigned long long)total, alpha);
  sign_pack_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(W), total / 8,
                                             packed);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_sign_to_i2s_launch(const uint8_t* sign, int64_t nbytes, uint8_t* codes,
                                        int num_sms, cudaStream_t stream) {
  int grid = num_sms * 4;
  const int64_t need = (nbytes + 255) / 256;
  if (need < grid) grid = (int)(need > 0 ? need : 1);
  sign_to_i2s_kernel<<<grid, 256, 0, stream>>>(sign, nbytes, codes);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_pack_launch(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                 float* gamma, void* workspace, cudaStream_t stream,
                                 int num_sms) {
  static_assert(sizeof(PackWs) <= 4096, "pack workspace");
  PackWs* ws = reinterpret_cast<PackWs*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(PackWs), stream) != cudaSuccess) return BITNET_ERR_CUDA;
  const int64_t total = N * K;
  const int64_t n4 = total / 4;
  int grid = num_sms * 4;
  const int64_t need = (n4 + 255) / 256;
  if (need < grid) grid = (int)(need > 0 ? need : 1);
  gamma_bucket_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(W), n4, ws);
  gamma_finalize_kernel<<<1, 32, 0, stream>>>(ws, (unsigned long long)total, gamma);
  ternary_pack_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(W), n4, ws,
                                                packed);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}
