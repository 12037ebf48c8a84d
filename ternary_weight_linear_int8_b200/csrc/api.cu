// C ABI of the library: argument validation, planning (which kernel, how
// much workspace) and dispatch.  Declarations and the contract of every entry
// point are in include/bitnet.h.
#include <cuda_runtime.h>

#include "common.cuh"

using namespace bitnet;

// Defined in the kernel sources of this translation unit.
size_t bitnet_pack_workspace_size_impl();
bitnet_status bitnet_pack_launch(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                 float* gamma, void* workspace, cudaStream_t stream, int num_sms);
bitnet_status bitnet_quant_launch(const void* src, bool src_f32, const float* gain, int64_t M,
                                  int64_t K, int8_t* xq, int64_t ld_q, bool perm, float* scale,
                                  int32_t* rowsum, double* sumsq, int8_t* xq_natural,
                                  cudaStream_t stream, const float* amax_in, float* amax_out,
                                  void* zero, size_t zero_bytes);
bitnet_status bitnet_decode_launch(const DecodeOp& op, int M, int num_sms, cudaStream_t stream);
bool bitnet_resident_fits(int fmt, int64_t M, int64_t N, int64_t K, int num_sms);
bool bitnet_resident_a48_fits(int64_t N, int64_t K, int num_sms);
bitnet_status bitnet_resident_a48_launch(const uint8_t* w, const float* gamma, int N, int K,
                                         const uint16_t* x, int n_out, const int8_t* rows,
                                         const float* scale, const int32_t* rowsum, uint16_t* y,
                                         float* y_f32, int32_t* acc4, int32_t* acc8,
                                         int num_sms, cudaStream_t stream);
bitnet_status bitnet_resident_launch(int fmt, const uint8_t* w, const float* gamma, int N, int K,
                                     const uint16_t* x, int M, uint16_t* y, float* y_f32,
                                     int32_t* acc, int num_sms, cudaStream_t stream);
bitnet_status bitnet_pack_w1_launch(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                    float* alpha, void* workspace, cudaStream_t stream,
                                    int num_sms);
bitnet_status bitnet_sign_to_i2s_launch(const uint8_t* sign, int64_t nbytes, uint8_t* codes,
                                        int num_sms, cudaStream_t stream);
bitnet_status bitnet_a48_quant_launch(const uint16_t* x, int64_t M, int64_t K, int64_t n_out,
                                      int8_t* rows, float* scale, int32_t* rowsum, int8_t* q4n,
                                      int8_t* q8n, float* s4, float* s8, cudaStream_t stream,
                                      void* zero, size_t zero_bytes);
bitnet_status bitnet_a48_combine_launch(const int32_t* acc2, const float* scale,
                                        const float* gamma, int64_t M, int64_t N, uint16_t* y,
                                        float* y_f32, int32_t* acc4, int32_t* acc8, int num_sms,
                                        cudaStream_t stream);
bitnet_status bitnet_gemm_launch(int mode, const int8_t* xq, const uint8_t* w0,
                                 const uint8_t* w1, GemmArgs a, int bn, int num_sms,
                                 cudaStream_t stream);
int bitnet_gemm_pick_bn(int M, int N, int num_sms);
int bitnet_batched_splits(int64_t M, int64_t N, int64_t K, int num_sms);
bitnet_status bitnet_batched_launch(const uint8_t* w, const float* gamma, int N, int K,
                                    const uint16_t* x, int M, uint16_t* y, float* y_f32,
                                    int32_t* acc, const float* amax_in, unsigned* amax_out,
                                    float* amax_clear, int32_t* ws_acc, int ldw,
                                    unsigned* ws_cnt, int num_sms, cudaStream_t stream);
bitnet_status bitnet_batched_prep_launch(const uint16_t* x, int M, int K, float* amax,
                                         void* zero, size_t zero_bytes, int num_sms,
                                         cudaStream_t stream);

namespace {

// Ragged K (K % 64 != 0): one thread per output, natural-layout x_q.
__global__ void __launch_bounds__(256) generic_linear_kernel(const uint8_t* __restrict__ packed,
                                                             const float* __restrict__ gamma,
                                                             int N, int K, int M,
                                                             const int8_t* __restrict__ xq,
                                                             const float* __restrict__ scale,
                                                             uint16_t* y, float* y_f32,
                                                             int32_t* acc_out) {
  pdl_wait();
  const int64_t total = (int64_t)M * N;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(o / N), n = (int)(o % N);
    const uint8_t* row = packed + (int64_t)n * (K / 4);
    const int8_t* xr = xq + (int64_t)m * K;
    int acc = 0;
    for (int k = 0; k < K; ++k) {
      const int code = (row[k >> 2] >> (2 * (k & 3))) & 3;
      acc += (int)xr[k] * (code - 1);
    }
    const float y32 = __fmul_rn(__int2float_rn(acc), __fdiv_rn(*gamma, scale[m]));
    y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
    if (y_f32) y_f32[o] = y32;
    if (acc_out) acc_out[o] = acc;
  }
}

// Last step of the tensor-parallel FFN: the all-reduced integer accumulators
// of the down projection dequantised with the all-reduced statistics, in the
// same steps as the single-GPU block: s2 = 127 / max(amax2, 1e-5),
// r1 = 1/sqrt(sum x^2 / H + eps), r2 = 1/sqrt(r1^6 sum h'^2 / I + eps) (fp64),
// y32 = (fp32(acc) * (gamma_d / s2)) * fp32(r1^3 r2).
__global__ void __launch_bounds__(256) ffn_tp_finish_kernel(
    const int32_t* __restrict__ acc, int M, int H, int I, const float* gamma_d,
    const float* __restrict__ amax2, const double* __restrict__ ssx,
    const double* __restrict__ ssh, float eps, uint16_t* y, float* y_f32) {
  pdl_wait();
  const int64_t total = (int64_t)M * H;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(o / H);
    const float d0 = __fdiv_rn(*gamma_d, qscale(amax2[m]));
    const double e = (double)eps;
    const double r1 = 1.0 / sqrt(ssx[m] / (double)H + e);
    const double r1_3 = r1 * r1 * r1;
    const double r2 = 1.0 / sqrt(r1_3 * r1_3 * (ssh[m] / (double)I) + e);
    const float f = (float)(r1_3 * r2);
    const float y32 = __fmul_rn(__fmul_rn(__int2float_rn(acc[o]), d0), f);
    y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(y32));
    if (y_f32) y_f32[o] = y32;
  }
}

struct DevInfo {
  int num_sms = 0;
  int major = 0;
};

// Per-device attributes, cached; an entry packs (major << 16) | SM count into
// one atomic word, so concurrent host threads read either 0 (not yet known,
// each queries it) or a complete entry.
bitnet_status device_info(DevInfo* out) {
  static std::atomic<uint32_t> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITNET_ERR_CUDA;
  if (dev < 0 || dev >= 64) return BITNET_ERR_UNSUPPORTED;
  uint32_t v = cache[dev].load(std::memory_order_acquire);
  if (v == 0) {
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return BITNET_ERR_CUDA;
    v = ((uint32_t)major << 16) | ((uint32_t)sms & 0xffffu);
    cache[dev].store(v, std::memory_order_release);
  }
  out->num_sms = (int)(v & 0xffffu);
  out->major = (int)(v >> 16);
  if (out->major != 10) return BITNET_ERR_UNSUPPORTED;
  return BITNET_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

// Which kernel serves bitnet_linear for this shape.
enum LinearPath { kPathGemv = 0, kPathGemm = 1, kPathGeneric = 2 };

int gemv_mpad(int64_t M) {
  const int64_t MT = M == 1 ? 1 : (M == 2 ? 2 : 4);
  return (int)(((M + MT - 1) / MT) * MT);
}

bool gemv_fits(int64_t M, int64_t K) {
  return M <= 8 && K % 64 == 0 && (int64_t)gemv_mpad(M) * K <= 65536;
}

LinearPath linear_path(int64_t M, int64_t K) {
  if (K % 64 != 0) return kPathGeneric;
  if (gemv_fits(M, K)) return kPathGemv;
  return kPathGemm;
}

// Split K over CTAs when the tile grid would leave most SMs idle.
int plan_ksplit(int64_t M, int64_t N, int64_t K, int bn, int num_sms) {
  if (M > 256) return 1;
  const int64_t tiles = ((N + 127) / 128) * ((M + bn - 1) / bn);
  const int64_t kst = (K + 127) / 128;
  if (tiles * 2 > num_sms) return 1;
  int64_t ks = num_sms / tiles;
  if (ks > 8) ks = 8;
  if (ks > kst / 2) ks = kst / 2;
  return ks < 1 ? 1 : (int)ks;
}

// Split-K scratch of the tensor-core path: the integer accumulators [M,N]
// followed by one counter per (128-feature, token) tile (tiles are at least
// 32 tokens wide); both are cleared before each launch.
size_t splitk_acc_bytes(int64_t M, int64_t N) { return al256((size_t)M * N * 4); }
size_t splitk_cnt_bytes(int64_t M, int64_t N) {
  return al256((size_t)((N + 127) / 128) * (size_t)((M + 31) / 32) * 4);
}

// Scratch of the batched decode kernel (4..64 tokens): per-token absmax
// slots -- slot 2 is filled from x by the prep kernel, slots 0 and 1 with slot
// 2 form the hand-over ring of a chain -- then one arrival counter per row
// group (at most 256 groups) and the split-K sums [M, ldw].  Everything after slot 2 is zeroed by
// the prep kernel and left zero by the layers.
struct BatchedWs {
  size_t slot[3], cnt, acc, total;
  int64_t ldw;
};

// Token counts the batched decode kernel serves.  Measured on the 2B decode
// chain it beats the streaming decode kernel's matrix-multiply items from 9
// tokens on and the tensor-core GEMM path up to 32 tokens; outside that range
// those paths stay.
bool batched_shape(int64_t M, int64_t K) { return M >= 9 && M <= 32 && K % 64 == 0; }

BatchedWs batched_ws_layout(int64_t M, int64_t N) {
  BatchedWs w{};
  const size_t a = al256((size_t)M * 4);
  w.slot[2] = 0;
  w.slot[0] = a;
  w.slot[1] = 2 * a;
  w.cnt = 3 * a;
  w.ldw = ((N + 16 * 256 + 3) / 4) * 4;     // at most 256 row groups, each padded to 16
  w.acc = w.cnt + al256(256 * 4);
  w.total = w.acc + al256((size_t)M * (size_t)w.ldw * 4);
  return w;
}

struct LinearWs {
  size_t xq, scale, rowsum, acc, total;
};

LinearWs linear_ws_layout(int64_t M, int64_t N, int64_t K) {
  LinearWs w{};
  const LinearPath p = linear_path(M, K);
  const size_t bt = batched_shape(M, K) ? batched_ws_layout(M, N).total : 0;
  if (p == kPathGemv) {
    w.total = bt;
    return w;
  }
  w.xq = 0;
  w.scale = al256((size_t)M * K);
  w.rowsum = w.scale + al256((size_t)M * 4);
  w.acc = w.rowsum + al256((size_t)M * 4);
  w.total = w.acc;
  // split-K accumulators are reserved for every small-M tensor-core shape
  if (p == kPathGemm && M <= 256) w.total = w.acc + splitk_acc_bytes(M, N) + splitk_cnt_bytes(M, N);
  if (bt > w.total) w.total = bt;
  return w;
}

struct FfnWs {
  bool gemv;
  size_t h, xq1, s1, rs1, ss1, xq2, s2, rs2, ss2, acc0, acc1, total;
};

FfnWs ffn_ws_layout(int64_t M, int64_t H, int64_t I) {
  FfnWs w{};
  w.gemv = gemv_fits(M, H) && gemv_fits(M, I);
  size_t off = 0;
  w.h = off;
  off += al256((size_t)M * I * 4);
  if (!w.gemv) {
    w.xq1 = off; off += al256((size_t)M * H);
    w.s1 = off; off += al256((size_t)M * 4);
    w.rs1 = off; off += al256((size_t)M * 4);
    w.ss1 = off; off += al256((size_t)M * 8);
    w.xq2 = off; off += al256((size_t)M * I);
    w.s2 = off; off += al256((size_t)M * 4);
    w.rs2 = off; off += al256((size_t)M * 4);
    w.ss2 = off; off += al256((size_t)M * 8);
    if (M <= 256) {   // split-K accumulators: gate (and later down), up
      const int64_t HI = H > I ? H : I;
      w.acc0 = off; off += splitk_acc_bytes(M, HI) + splitk_cnt_bytes(M, HI);
      w.acc1 = off; off += al256((size_t)M * I * 4);
    }
  }
  w.total = off;
  return w;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Workspace of bitnet_linear_a48: the 2M code rows (q4 of token m at row 2m,
// q8 at 2m + 1, kernel K order), their scales and row sums, the exact
// accumulators of the 2M rows, the tensor-core kernel's (unused) bf16 rows,
// and its split-K accumulators for small M.
struct A48Ws {
  size_t rows, scale, rowsum, acc2, yscr, acc, total;
};

// Workspace of the tensor-parallel FFN steps on one shard of Ir intermediate
// features: first-norm codes of x (gate/up step) or second-norm codes of h'
// (down step), their scales and row sums, the statistics pass's codes, the
// down step's unused bf16 rows, and the tensor-core kernel's split-K
// accumulators (gate and up, or down).
struct TpWs {
  size_t xq, s, rs, xq2, s2, yscr, acc0, acc1, total;
};

TpWs tp_ws_layout(int64_t M, int64_t H, int64_t Ir) {
  TpWs w{};
  const int64_t HI = H > Ir ? H : Ir;
  size_t off = 0;
  w.xq = off; off += al256((size_t)M * HI);
  w.s = off; off += al256((size_t)M * 4);
  w.rs = off; off += al256((size_t)M * 4);
  w.xq2 = off; off += al256((size_t)M * Ir);
  w.s2 = off; off += al256((size_t)M * 4);
  w.yscr = off; off += al256((size_t)M * H * 2);
  w.acc0 = off;
  if (M <= 256) {
    off += splitk_acc_bytes(M, HI) + splitk_cnt_bytes(M, HI);
    w.acc1 = off;
    off += al256((size_t)M * Ir * 4);
  }
  w.total = off;
  return w;
}

A48Ws a48_ws_layout(int64_t M, int64_t N, int64_t K) {
  A48Ws w{};
  const int64_t M2 = 2 * M;
  size_t off = 0;
  w.rows = off; off += al256((size_t)M2 * K);
  w.scale = off; off += al256((size_t)M2 * 4);
  w.rowsum = off; off += al256((size_t)M2 * 4);
  w.acc2 = off; off += al256((size_t)M2 * N * 4);
  w.yscr = off; off += al256((size_t)M2 * N * 2);
  w.acc = off;
  if (M2 <= 256) off += splitk_acc_bytes(M2, N) + splitk_cnt_bytes(M2, N);
  w.total = off;
  return w;
}

}  // namespace

extern "C" {

const char* bitnet_status_string(int status) {
  switch (status) {
    case BITNET_OK: return "BITNET_OK";
    case BITNET_ERR_INVALID_ARG: return "BITNET_ERR_INVALID_ARG";
    case BITNET_ERR_SHAPE: return "BITNET_ERR_SHAPE";
    case BITNET_ERR_ALIGN: return "BITNET_ERR_ALIGN";
    case BITNET_ERR_WORKSPACE: return "BITNET_ERR_WORKSPACE";
    case BITNET_ERR_UNSUPPORTED: return "BITNET_ERR_UNSUPPORTED";
    case BITNET_ERR_CUDA: return "BITNET_ERR_CUDA";
    case BITNET_ERR_TIMEOUT: return "BITNET_ERR_TIMEOUT";
    case BITNET_ERR_NONFINITE: return "BITNET_ERR_NONFINITE";
    default: return "BITNET_ERR_UNKNOWN";
  }
}

int bitnet_version(void) { return 100; }

size_t bitnet_pack_workspace_size(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return bitnet_pack_workspace_size_impl();
}

bitnet_status bitnet_pack_weights(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                  float* gamma, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!W || !packed || !gamma) return BITNET_ERR_INVALID_ARG;
  if (N < 1 || K < 4 || K % 4 != 0 || N > (int64_t(1) << 39) / K) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || ((uintptr_t)gamma & 3u)) return BITNET_ERR_ALIGN;
  if (!workspace || workspace_bytes < bitnet_pack_workspace_size(N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  return bitnet_pack_launch(W, N, K, packed, gamma, workspace, as_stream(stream), d.num_sms);
}

bitnet_status bitnet_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* scale,
                               int32_t* rowsum, void* stream) {
  if (!x || !xq || !scale) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || K < 4 || K % 4 != 0 || M > 0x7fffffff || K > (int64_t(1) << 31))
    return BITNET_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(xq) || ((uintptr_t)scale & 3u) || ((uintptr_t)rowsum & 3u))
    return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  return bitnet_quant_launch(x, false, nullptr, M, K, xq, K, false, scale, rowsum, nullptr,
                             nullptr, as_stream(stream));
}

size_t bitnet_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 4) return 0;
  return linear_ws_layout(M, N, K).total;
}

}  // extern "C"

namespace {

// Enqueue one validated BitLinear.
bitnet_status linear_enqueue(const uint8_t* packed, const float* gamma, int64_t N, int64_t K,
                             const uint16_t* x, int64_t M, uint16_t* y, float* y_f32,
                             int32_t* acc, void* workspace, const LinearWs& L, const DevInfo& d,
                             cudaStream_t s) {
  bitnet_status st = BITNET_OK;
  const LinearPath p = linear_path(M, K);
  const int bsplit = batched_shape(M, K) ? bitnet_batched_splits(M, N, K, d.num_sms) : 0;
  if (bsplit > 0) {
    // absmax of x (and a cleared split-K scratch), then the batched kernel
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const BatchedWs b = batched_ws_layout(M, N);
    float* amax = reinterpret_cast<float*>(ws + b.slot[2]);
    st = bitnet_batched_prep_launch(x, (int)M, (int)K, amax, ws + b.cnt,
                                    bsplit > 1 ? b.total - b.cnt : 0, d.num_sms, s);
    if (st != BITNET_OK) return st;
    return bitnet_batched_launch(packed, gamma, (int)N, (int)K, x, (int)M, y, y_f32, acc, amax,
                                 nullptr, nullptr, reinterpret_cast<int32_t*>(ws + b.acc),
                                 (int)b.ldw, reinterpret_cast<unsigned*>(ws + b.cnt), d.num_sms,
                                 s);
  }
  if (p == kPathGemv) {
    if (bitnet_resident_fits(0, M, N, K, d.num_sms))
      return bitnet_resident_launch(0, packed, gamma, (int)N, (int)K, x, (int)M, y, y_f32, acc,
                                    d.num_sms, s);
    DecodeOp a{};
    a.mode = kLinear;
    a.w0 = packed; a.gamma0 = gamma;
    a.N = (int)N; a.K = (int)K;
    a.x = x;
    a.y = y; a.y_f32 = y_f32; a.acc0 = acc;
    return bitnet_decode_launch(a, (int)M, d.num_sms, s);
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
  float* sc = reinterpret_cast<float*>(ws + L.scale);
  int32_t* rs = reinterpret_cast<int32_t*>(ws + L.rowsum);
  if (p == kPathGeneric) {
    st = bitnet_quant_launch(x, false, nullptr, M, K, xq, K, false, sc, rs, nullptr, nullptr, s);
    if (st != BITNET_OK) return st;
    int64_t blocks = (M * N + 255) / 256;
    if (blocks > (int64_t)d.num_sms * 16) blocks = (int64_t)d.num_sms * 16;
    generic_linear_kernel<<<(unsigned)blocks, 256, 0, s>>>(packed, gamma, (int)N, (int)K, (int)M,
                                                          xq, sc, y, y_f32, acc);
    return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
  }
  const int bn = bitnet_gemm_pick_bn((int)M, (int)N, d.num_sms);
  GemmArgs a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K;
  a.ksplit = plan_ksplit(M, N, K, bn, d.num_sms);
  a.scale = sc; a.rowsum = rs; a.gamma0 = gamma;
  a.y = y; a.y_f32 = y_f32; a.acc0 = acc;
  if (a.ksplit > 1) {
    a.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc);
    a.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc + splitk_acc_bytes(M, N));
  }
  // the quantiser also clears the split-K accumulators and tile counters
  // (after its dependency wait; the GEMM adds into them only after its own)
  st = bitnet_quant_launch(x, false, nullptr, M, K, xq, K, true, sc, rs, nullptr, nullptr, s,
                           nullptr, nullptr, a.ksplit > 1 ? a.acc_ws0 : nullptr,
                           a.ksplit > 1 ? splitk_acc_bytes(M, N) + splitk_cnt_bytes(M, N) : 0);
  if (st != BITNET_OK) return st;
  return bitnet_gemm_launch(0 /*linear*/, xq, packed, nullptr, a, bn, d.num_sms, s);
}

}  // namespace

extern "C" {

bitnet_status bitnet_linear(const uint8_t* packed, const float* gamma, int64_t N, int64_t K,
                            const uint16_t* x, int64_t M, uint16_t* y, float* y_f32,
                            int32_t* acc, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!packed || !gamma || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 4 || K % 4 != 0 || K > 524288 || M > 0x7fffffff || N > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || ((uintptr_t)gamma & 3u) ||
      ((uintptr_t)y_f32 & 3u) || ((uintptr_t)acc & 3u))
    return BITNET_ERR_ALIGN;
  const LinearWs L = linear_ws_layout(M, N, K);
  if (L.total > 0) {
    if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  }
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  return linear_enqueue(packed, gamma, N, K, x, M, y, y_f32, acc, workspace, L, d,
                        as_stream(stream));
}

size_t bitnet_ffn_workspace_size(int64_t M, int64_t H, int64_t I) {
  if (M < 1 || H < 1 || I < 1) return 0;
  return ffn_ws_layout(M, H, I).total;
}

bitnet_status bitnet_ffn(const uint16_t* x, int64_t M, int64_t H, int64_t I,
                         const float* norm1_w, const uint8_t* gate, const float* gamma_gate,
                         const uint8_t* up, const float* gamma_up, const float* norm2_w,
                         const uint8_t* down, const float* gamma_down, float eps, uint16_t* y,
                         const bitnet_ffn_debug* debug, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (!x || !gate || !gamma_gate || !up || !gamma_up || !down || !gamma_down || !y)
    return BITNET_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || H < 64 || I < 64 || H % 64 != 0 || I % 64 != 0 || H > 524288 || I > 524288 ||
      M > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y) || !aligned16(gate) || !aligned16(up) || !aligned16(down))
    return BITNET_ERR_ALIGN;
  const FfnWs L = ffn_ws_layout(M, H, I);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  bitnet_ffn_debug dbg{};
  if (debug) dbg = *debug;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* h = reinterpret_cast<float*>(ws + L.h);
  if (L.gemv) {
    // two decode launches: gate/up (h'), then down; the down kernel streams
    // its weights while gate/up finishes (programmatic dependent launch)
    DecodeOp g{};
    g.mode = kGlu;
    g.w0 = gate; g.gamma0 = gamma_gate; g.w1 = up; g.gamma1 = gamma_up;
    g.N = (int)I; g.K = (int)H;
    g.x = x; g.gain = norm1_w;
    g.h = dbg.h ? dbg.h : h;
    g.acc0 = dbg.acc_gate; g.acc1 = dbg.acc_up; g.xq_dbg = dbg.xq1;
    st = bitnet_decode_launch(g, (int)M, d.num_sms, s);
    if (st != BITNET_OK) return st;
    DecodeOp dn{};
    dn.mode = kDown;
    dn.w0 = down; dn.gamma0 = gamma_down;
    dn.N = (int)H; dn.K = (int)I;
    dn.x = g.h; dn.gain = norm2_w; dn.xnorm = x; dn.H = (int)H; dn.eps = eps;
    dn.y = y; dn.y_f32 = dbg.y_f32; dn.acc0 = dbg.acc_down; dn.xq_dbg = dbg.xq2;
    return bitnet_decode_launch(dn, (int)M, d.num_sms, s);
  }
  int8_t* xq1 = reinterpret_cast<int8_t*>(ws + L.xq1);
  float* s1 = reinterpret_cast<float*>(ws + L.s1);
  int32_t* rs1 = reinterpret_cast<int32_t*>(ws + L.rs1);
  double* ss1 = reinterpret_cast<double*>(ws + L.ss1);
  int8_t* xq2 = reinterpret_cast<int8_t*>(ws + L.xq2);
  float* s2 = reinterpret_cast<float*>(ws + L.s2);
  int32_t* rs2 = reinterpret_cast<int32_t*>(ws + L.rs2);
  double* ss2 = reinterpret_cast<double*>(ws + L.ss2);
  float* hbuf = dbg.h ? dbg.h : h;
  // gate and up share the activation tile: keep it at the full 256 tokens
  const int bn = M > 128 ? 256 : bitnet_gemm_pick_bn((int)M, (int)I, d.num_sms);
  GemmArgs g{};
  g.M = (int)M; g.N = (int)I; g.K = (int)H;
  g.ksplit = plan_ksplit(M, I, H, bn, d.num_sms);
  g.scale = s1; g.rowsum = rs1; g.gamma0 = gamma_gate; g.gamma1 = gamma_up;
  g.h = hbuf; g.acc0 = dbg.acc_gate; g.acc1 = dbg.acc_up;
  if (g.ksplit > 1) {
    g.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc0);
    g.acc_ws1 = reinterpret_cast<int32_t*>(ws + L.acc1);
    g.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc0 + splitk_acc_bytes(M, I));
  }
  // each quantiser also clears the split-K scratch of the GEMM after it
  st = bitnet_quant_launch(x, false, norm1_w, M, H, xq1, H, true, s1, rs1, ss1, dbg.xq1, s,
                           nullptr, nullptr, g.ksplit > 1 ? ws + L.acc0 : nullptr,
                           g.ksplit > 1 ? (L.acc1 - L.acc0) + al256((size_t)M * I * 4) : 0);
  if (st != BITNET_OK) return st;
  st = bitnet_gemm_launch(1 /*glu*/, xq1, gate, up, g, bn, d.num_sms, s);
  if (st != BITNET_OK) return st;
  GemmArgs dn{};
  const int bn_d = bitnet_gemm_pick_bn((int)M, (int)H, d.num_sms);
  dn.M = (int)M; dn.N = (int)H; dn.K = (int)I;
  dn.ksplit = plan_ksplit(M, H, I, bn_d, d.num_sms);
  dn.scale = s2; dn.rowsum = rs2; dn.gamma0 = gamma_down;
  dn.sumsq_h = ss2; dn.sumsq_x = ss1; dn.H = (int)H; dn.eps = eps;
  dn.y = y; dn.y_f32 = dbg.y_f32; dn.acc0 = dbg.acc_down;
  if (dn.ksplit > 1) {
    dn.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc0);
    dn.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc0 + splitk_acc_bytes(M, H));
  }
  st = bitnet_quant_launch(hbuf, true, norm2_w, M, I, xq2, I, true, s2, rs2, ss2, dbg.xq2, s,
                           nullptr, nullptr, dn.ksplit > 1 ? ws + L.acc0 : nullptr,
                           dn.ksplit > 1 ? splitk_acc_bytes(M, H) + splitk_cnt_bytes(M, H) : 0);
  if (st != BITNET_OK) return st;
  return bitnet_gemm_launch(2 /*down*/, xq2, down, nullptr, dn, bn_d, d.num_sms, s);
}

size_t bitnet_linear_chain_workspace_size(int64_t L, const int64_t* N, const int64_t* K,
                                          int64_t M) {
  if (L < 1 || !N || !K || M < 1) return 0;
  size_t lin = 0;   // the largest layer's bitnet_linear scratch (reused)
  for (int64_t l = 0; l < L; ++l) {
    if (N[l] < 1 || K[l] < 4) return 0;
    const size_t b = linear_ws_layout(M, N[l], K[l]).total;
    if (b > lin) lin = b;
  }
  return lin;
}

bitnet_status bitnet_linear_chain(int64_t L, const uint8_t* const* packed,
                                  const float* const* gamma, const int64_t* N, const int64_t* K,
                                  const uint16_t* x, int64_t M, uint16_t* const* y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (L < 1 || !packed || !gamma || !N || !K || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7fffffff) return BITNET_ERR_SHAPE;
  if (!aligned16(x)) return BITNET_ERR_ALIGN;
  for (int64_t l = 0; l < L; ++l) {
    if (!packed[l] || !gamma[l] || !y[l]) return BITNET_ERR_INVALID_ARG;
    if (N[l] < 1 || K[l] < 4 || K[l] % 4 != 0 || K[l] > 524288 || N[l] > 0x7fffffff)
      return BITNET_ERR_SHAPE;
    if (l > 0 && K[l] != N[l - 1]) return BITNET_ERR_SHAPE;
    if (!aligned16(packed[l]) || !aligned16(y[l]) || ((uintptr_t)gamma[l] & 3u))
      return BITNET_ERR_ALIGN;
    // a layer's output may not overlap its own input (the CTAs of one
    // launch read the input while others already write the output)
    const uintptr_t in = reinterpret_cast<uintptr_t>(l == 0 ? x : y[l - 1]);
    const uintptr_t out = reinterpret_cast<uintptr_t>(y[l]);
    const uintptr_t in_end = in + (uintptr_t)(M * K[l] * 2);
    const uintptr_t out_end = out + (uintptr_t)(M * N[l] * 2);
    if (in < out_end && out < in_end) return BITNET_ERR_INVALID_ARG;
  }
  const size_t need = bitnet_linear_chain_workspace_size(L, N, K, M);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  }
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  const cudaStream_t s = as_stream(stream);
  // 4..64 tokens on layers that all fit the batched decode kernel: one absmax
  // pass over x, then one launch per layer, each handing its outputs' per-token
  // absmax to the next through a ring of three slots (layer l reads slot
  // (l + 2) % 3, folds its own into slot l % 3 and clears slot (l + 1) % 3,
  // which the layer before it has finished reading)
  bool batched = batched_shape(M, K[0]);
  bool any_split = false;
  int64_t n_max = 0;
  for (int64_t l = 0; batched && l < L; ++l) {
    const int sp = bitnet_batched_splits(M, N[l], K[l], d.num_sms);
    batched = sp > 0;
    any_split = any_split || sp > 1;
    if (N[l] > n_max) n_max = N[l];
  }
  if (batched) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const BatchedWs b = batched_ws_layout(M, n_max);
    float* slot[3];
    for (int i = 0; i < 3; ++i) slot[i] = reinterpret_cast<float*>(ws + b.slot[i]);
    st = bitnet_batched_prep_launch(x, (int)M, (int)K[0], slot[2], ws + b.slot[0],
                                    (any_split ? b.total : b.acc) - b.slot[0], d.num_sms, s);
    if (st != BITNET_OK) return st;
    for (int64_t l = 0; l < L; ++l) {
      const bool last = l + 1 == L;
      st = bitnet_batched_launch(
          packed[l], gamma[l], (int)N[l], (int)K[l], l == 0 ? x : y[l - 1], (int)M, y[l],
          nullptr, nullptr, slot[(l + 2) % 3],
          last ? nullptr : reinterpret_cast<unsigned*>(slot[l % 3]),
          last ? nullptr : slot[(l + 1) % 3], reinterpret_cast<int32_t*>(ws + b.acc),
          (int)b.ldw, reinterpret_cast<unsigned*>(ws + b.cnt), d.num_sms, s);
      if (st != BITNET_OK) return st;
    }
    return BITNET_OK;
  }
  // otherwise one launch per layer, in order on the stream (validated above,
  // planned here); each decode kernel starts loading its weights while the
  // layer before it finishes
  for (int64_t l = 0; l < L; ++l) {
    const LinearWs lw = linear_ws_layout(M, N[l], K[l]);
    st = linear_enqueue(packed[l], gamma[l], N[l], K[l], l == 0 ? x : y[l - 1], M, y[l], nullptr,
                        nullptr, workspace, lw, d, s);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

}  // extern "C"

namespace {

// Scratch of bitnet_linear_multi.  On the tensor-core path (shared codes):
// the codes, scales and row sums of x once, then for tokens <= 256 one
// split-K region (accumulators + tile counters) per matrix, all cleared by
// the one quantiser launch.  Otherwise the largest matrix's bitnet_linear
// scratch, reused by each call in turn.
struct MultiWs {
  bool shared;
  size_t xq, scale, rowsum, acc, total;
};

MultiWs multi_ws_layout(int64_t L, const int64_t* N, int64_t K, int64_t M) {
  MultiWs w{};
  w.shared = linear_path(M, K) == kPathGemm && !batched_shape(M, K);
  if (!w.shared) {
    for (int64_t l = 0; l < L; ++l) {
      const size_t b = linear_ws_layout(M, N[l], K).total;
      if (b > w.total) w.total = b;
    }
    return w;
  }
  w.xq = 0;
  w.scale = al256((size_t)M * K);
  w.rowsum = w.scale + al256((size_t)M * 4);
  w.acc = w.rowsum + al256((size_t)M * 4);
  w.total = w.acc;
  if (M <= 256)
    for (int64_t l = 0; l < L; ++l) w.total += splitk_acc_bytes(M, N[l]) + splitk_cnt_bytes(M, N[l]);
  return w;
}

}  // namespace

extern "C" {

size_t bitnet_linear_multi_workspace_size(int64_t L, const int64_t* N, int64_t K, int64_t M) {
  if (L < 1 || !N || M < 1 || K < 4) return 0;
  for (int64_t l = 0; l < L; ++l)
    if (N[l] < 1) return 0;
  return multi_ws_layout(L, N, K, M).total;
}

bitnet_status bitnet_linear_multi(int64_t L, const uint8_t* const* packed,
                                  const float* const* gamma, const int64_t* N, int64_t K,
                                  const uint16_t* x, int64_t M, uint16_t* const* y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (L < 1 || !packed || !gamma || !N || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7fffffff || K < 4 || K % 4 != 0 || K > 524288) return BITNET_ERR_SHAPE;
  if (!aligned16(x)) return BITNET_ERR_ALIGN;
  const uintptr_t in = reinterpret_cast<uintptr_t>(x);
  const uintptr_t in_end = in + (uintptr_t)(M * K * 2);
  for (int64_t l = 0; l < L; ++l) {
    if (!packed[l] || !gamma[l] || !y[l]) return BITNET_ERR_INVALID_ARG;
    if (N[l] < 1 || N[l] > 0x7fffffff) return BITNET_ERR_SHAPE;
    if (!aligned16(packed[l]) || !aligned16(y[l]) || ((uintptr_t)gamma[l] & 3u))
      return BITNET_ERR_ALIGN;
    // no output may overlap the input (read by every matrix) or another output
    const uintptr_t out = reinterpret_cast<uintptr_t>(y[l]);
    const uintptr_t out_end = out + (uintptr_t)(M * N[l] * 2);
    if (in < out_end && out < in_end) return BITNET_ERR_INVALID_ARG;
    for (int64_t j = 0; j < l; ++j) {
      const uintptr_t o2 = reinterpret_cast<uintptr_t>(y[j]);
      const uintptr_t o2_end = o2 + (uintptr_t)(M * N[j] * 2);
      if (o2 < out_end && out < o2_end) return BITNET_ERR_INVALID_ARG;
    }
  }
  const MultiWs W = multi_ws_layout(L, N, K, M);
  if (W.total > 0) {
    if (!workspace || workspace_bytes < W.total) return BITNET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  }
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if (!W.shared) {
    // decode and generic paths quantise inside their own kernels: one
    // bitnet_linear per matrix, in order on the stream
    for (int64_t l = 0; l < L; ++l) {
      st = linear_enqueue(packed[l], gamma[l], N[l], K, x, M, y[l], nullptr, nullptr, workspace,
                          linear_ws_layout(M, N[l], K), d, s);
      if (st != BITNET_OK) return st;
    }
    return BITNET_OK;
  }
  // tensor-core path: one quantiser launch (which also clears every matrix's
  // split-K region), then one GEMM per matrix on the shared codes
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws + W.xq);
  float* sc = reinterpret_cast<float*>(ws + W.scale);
  int32_t* rs = reinterpret_cast<int32_t*>(ws + W.rowsum);
  st = bitnet_quant_launch(x, false, nullptr, M, K, xq, K, true, sc, rs, nullptr, nullptr, s,
                           nullptr, nullptr, W.total > W.acc ? ws + W.acc : nullptr,
                           W.total - W.acc);
  if (st != BITNET_OK) return st;
  size_t acc_off = W.acc;
  for (int64_t l = 0; l < L; ++l) {
    const int bn = bitnet_gemm_pick_bn((int)M, (int)N[l], d.num_sms);
    GemmArgs a{};
    a.M = (int)M; a.N = (int)N[l]; a.K = (int)K;
    a.ksplit = plan_ksplit(M, N[l], K, bn, d.num_sms);
    a.scale = sc; a.rowsum = rs; a.gamma0 = gamma[l];
    a.y = y[l];
    if (a.ksplit > 1) {
      a.acc_ws0 = reinterpret_cast<int32_t*>(ws + acc_off);
      a.tile_cnt = reinterpret_cast<int32_t*>(ws + acc_off + splitk_acc_bytes(M, N[l]));
    }
    if (M <= 256) acc_off += splitk_acc_bytes(M, N[l]) + splitk_cnt_bytes(M, N[l]);
    st = bitnet_gemm_launch(0 /*linear*/, xq, packed[l], nullptr, a, bn, d.num_sms, s);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

size_t bitnet_pack_w1_workspace_size(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return bitnet_pack_workspace_size_impl();
}

bitnet_status bitnet_pack_weights_w1(const float* W, int64_t N, int64_t K, uint8_t* packed,
                                     float* alpha, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!W || !packed || !alpha) return BITNET_ERR_INVALID_ARG;
  if (N < 1 || K < 8 || K % 8 != 0 || N > (int64_t(1) << 39) / K) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || ((uintptr_t)alpha & 3u)) return BITNET_ERR_ALIGN;
  if (!workspace || workspace_bytes < bitnet_pack_w1_workspace_size(N, K))
    return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  return bitnet_pack_w1_launch(W, N, K, packed, alpha, workspace, as_stream(stream), d.num_sms);
}

size_t bitnet_linear_w1_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 8) return 0;
  return al256((size_t)N * (size_t)(K / 4)) + linear_ws_layout(M, N, K).total;
}

bitnet_status bitnet_linear_w1(const uint8_t* packed, const float* alpha, int64_t N, int64_t K,
                               const uint16_t* x, int64_t M, uint16_t* y, float* y_f32,
                               int32_t* acc, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!packed || !alpha || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 8 || K % 8 != 0 || K > 524288 || M > 0x7fffffff || N > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || ((uintptr_t)alpha & 3u) ||
      ((uintptr_t)y_f32 & 3u) || ((uintptr_t)acc & 3u))
    return BITNET_ERR_ALIGN;
  const size_t need = bitnet_linear_w1_workspace_size(M, N, K);
  if (!workspace || workspace_bytes < need) return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  cudaStream_t s = as_stream(stream);
  // one to three tokens, packed rows a multiple of 16 bytes: the decode kernel
  // on the sign bits themselves
  if (K % 128 == 0 && bitnet_resident_fits(1, M, N, K, d.num_sms))
    return bitnet_resident_launch(1, packed, alpha, (int)N, (int)K, x, (int)M, y, y_f32, acc,
                                  d.num_sms, s);
  // otherwise the same +-1 matrix as ternary I2_S codes, then BitLinear with
  // gamma = alpha
  uint8_t* codes = static_cast<uint8_t*>(workspace);
  st = bitnet_sign_to_i2s_launch(packed, N * (K / 8), codes, d.num_sms, s);
  if (st != BITNET_OK) return st;
  const LinearWs L = linear_ws_layout(M, N, K);
  return linear_enqueue(codes, alpha, N, K, x, M, y, y_f32, acc,
                        codes + al256((size_t)N * (size_t)(K / 4)), L, d, s);
}

bitnet_status bitnet_linear_tl2(const uint8_t* packed, const float* gamma, int64_t N, int64_t K,
                                const uint16_t* x, uint16_t* y, float* y_f32, int32_t* acc,
                                void* stream) {
  if (!packed || !gamma || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (N < 1 || K < 64 || K % 64 != 0 || K > 524288 || N > 0x7fffffff) return BITNET_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || ((uintptr_t)gamma & 3u) ||
      ((uintptr_t)y_f32 & 3u) || ((uintptr_t)acc & 3u))
    return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  if (!bitnet_resident_fits(2, 1, N, K, d.num_sms)) return BITNET_ERR_UNSUPPORTED;
  return bitnet_resident_launch(2, packed, gamma, (int)N, (int)K, x, 1, y, y_f32, acc, d.num_sms,
                                as_stream(stream));
}

bitnet_status bitnet_quant_act_a48(const uint16_t* x, int64_t M, int64_t K, int64_t n_out,
                                   int8_t* q4, float* s4, int8_t* q8, float* s8, void* stream) {
  if (!x || !q4 || !s4 || !q8 || !s8) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || K < 8 || K % 8 != 0 || M > 0x7fffffff || K > 524288) return BITNET_ERR_SHAPE;
  if (n_out < 0 || n_out > K) return BITNET_ERR_INVALID_ARG;
  if (!aligned16(x) || ((uintptr_t)s4 & 3u) || ((uintptr_t)s8 & 3u)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  return bitnet_a48_quant_launch(x, M, K, n_out, nullptr, nullptr, nullptr, q4, q8, s4, s8,
                                 as_stream(stream), nullptr, 0);
}

size_t bitnet_linear_a48_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 8) return 0;
  return a48_ws_layout(M, N, K).total;
}

bitnet_status bitnet_linear_a48(const uint8_t* packed, const float* gamma, int64_t N, int64_t K,
                                const uint16_t* x, int64_t M, int64_t n_out, uint16_t* y,
                                float* y_f32, int32_t* acc4, int32_t* acc8, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!packed || !gamma || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || K > 524288 || M > 0x3fffffff ||
      N > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (n_out < 0 || n_out > K) return BITNET_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || ((uintptr_t)gamma & 3u) ||
      ((uintptr_t)y_f32 & 3u) || ((uintptr_t)acc4 & 3u) || ((uintptr_t)acc8 & 3u))
    return BITNET_ERR_ALIGN;
  const A48Ws L = a48_ws_layout(M, N, K);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* rows = reinterpret_cast<int8_t*>(ws + L.rows);
  float* sc = reinterpret_cast<float*>(ws + L.scale);
  int32_t* rs = reinterpret_cast<int32_t*>(ws + L.rowsum);
  int32_t* acc2 = reinterpret_cast<int32_t*>(ws + L.acc2);
  // one token whose weight slices fit shared memory: the resident kernel
  // quantises the token itself (every CTA) and combines the two code rows in
  // its epilogue; one launch
  if (M == 1 && bitnet_resident_a48_fits(N, K, d.num_sms))
    return bitnet_resident_a48_launch(packed, gamma, (int)N, (int)K, x, (int)n_out, nullptr,
                                      nullptr, nullptr, y, y_f32, acc4, acc8, d.num_sms, s);
  // the integer products of all 2M code rows on the tensor-core kernel
  const int64_t M2 = 2 * M;
  const int bn = bitnet_gemm_pick_bn((int)M2, (int)N, d.num_sms);
  GemmArgs a{};
  a.M = (int)M2; a.N = (int)N; a.K = (int)K;
  a.ksplit = plan_ksplit(M2, N, K, bn, d.num_sms);
  a.scale = sc; a.rowsum = rs; a.gamma0 = gamma;
  a.y = reinterpret_cast<uint16_t*>(ws + L.yscr);
  a.acc0 = acc2;
  if (a.ksplit > 1) {
    a.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc);
    a.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc + splitk_acc_bytes(M2, N));
  }
  // the quantiser also clears the GEMM's split-K scratch
  st = bitnet_a48_quant_launch(x, M, K, n_out, rows, sc, rs, nullptr, nullptr, nullptr, nullptr,
                               s, a.ksplit > 1 ? a.acc_ws0 : nullptr,
                               a.ksplit > 1 ? splitk_acc_bytes(M2, N) + splitk_cnt_bytes(M2, N)
                                            : 0);
  if (st != BITNET_OK) return st;
  st = bitnet_gemm_launch(0 /*linear*/, rows, packed, nullptr, a, bn, d.num_sms, s);
  if (st != BITNET_OK) return st;
  return bitnet_a48_combine_launch(acc2, sc, gamma, M, N, y, y_f32, acc4, acc8, d.num_sms, s);
}

size_t bitnet_ffn_tp_workspace_size(int64_t M, int64_t H, int64_t Ir) {
  if (M < 1 || H < 1 || Ir < 1) return 0;
  return tp_ws_layout(M, H, Ir).total;
}

bitnet_status bitnet_ffn_tp_gate_up(const uint16_t* x, int64_t M, int64_t H, int64_t Ir,
                                    const float* norm1_w, const uint8_t* gate,
                                    const float* gamma_gate, const uint8_t* up,
                                    const float* gamma_up, const float* norm2_w, float* h,
                                    float* amax2, double* sumsq_h, double* sumsq_x,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !gate || !gamma_gate || !up || !gamma_up || !h || !amax2 || !sumsq_h || !sumsq_x)
    return BITNET_ERR_INVALID_ARG;
  if (M < 1 || H < 64 || Ir < 64 || H % 64 != 0 || Ir % 64 != 0 || H > 524288 || Ir > 524288 ||
      M > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(h) || !aligned16(gate) || !aligned16(up) ||
      ((uintptr_t)amax2 & 3u) || ((uintptr_t)sumsq_h & 7u) || ((uintptr_t)sumsq_x & 7u))
    return BITNET_ERR_ALIGN;
  const TpWs L = tp_ws_layout(M, H, Ir);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq1 = reinterpret_cast<int8_t*>(ws + L.xq);
  float* s1 = reinterpret_cast<float*>(ws + L.s);
  int32_t* rs1 = reinterpret_cast<int32_t*>(ws + L.rs);
  const int bn = M > 128 ? 256 : bitnet_gemm_pick_bn((int)M, (int)Ir, d.num_sms);
  GemmArgs g{};
  g.M = (int)M; g.N = (int)Ir; g.K = (int)H;
  g.ksplit = plan_ksplit(M, Ir, H, bn, d.num_sms);
  g.scale = s1; g.rowsum = rs1; g.gamma0 = gamma_gate; g.gamma1 = gamma_up;
  g.h = h;
  if (g.ksplit > 1) {
    g.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc0);
    g.acc_ws1 = reinterpret_cast<int32_t*>(ws + L.acc1);
    g.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc0 + splitk_acc_bytes(M, Ir));
  }
  // every rank holds the whole token: the same codes on every shard (the
  // quantiser also clears the GEMM's split-K scratch)
  st = bitnet_quant_launch(x, false, norm1_w, M, H, xq1, H, true, s1, rs1, sumsq_x, nullptr, s,
                           nullptr, nullptr, g.ksplit > 1 ? ws + L.acc0 : nullptr,
                           g.ksplit > 1 ? (L.acc1 - L.acc0) + al256((size_t)M * Ir * 4) : 0);
  if (st != BITNET_OK) return st;
  st = bitnet_gemm_launch(1 /*glu*/, xq1, gate, up, g, bn, d.num_sms, s);
  if (st != BITNET_OK) return st;
  // this shard's statistics of h' * n2: absmax and sum of squares of h'
  return bitnet_quant_launch(h, true, norm2_w, M, Ir, reinterpret_cast<int8_t*>(ws + L.xq2), Ir,
                             false, reinterpret_cast<float*>(ws + L.s2), nullptr, sumsq_h,
                             nullptr, s, nullptr, amax2, nullptr, 0);
}

bitnet_status bitnet_ffn_tp_down(const float* h, int64_t M, int64_t H, int64_t Ir,
                                 const float* norm2_w, const uint8_t* down, const float* amax2,
                                 int32_t* acc, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!h || !down || !amax2 || !acc) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || H < 64 || Ir < 64 || H % 64 != 0 || Ir % 64 != 0 || H > 524288 || Ir > 524288 ||
      M > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (!aligned16(h) || !aligned16(down) || ((uintptr_t)amax2 & 3u) || ((uintptr_t)acc & 3u))
    return BITNET_ERR_ALIGN;
  const TpWs L = tp_ws_layout(M, H, Ir);
  if (!workspace || workspace_bytes < L.total) return BITNET_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq2 = reinterpret_cast<int8_t*>(ws + L.xq);
  float* s2 = reinterpret_cast<float*>(ws + L.s);
  int32_t* rs2 = reinterpret_cast<int32_t*>(ws + L.rs);
  // the shard's h' * n2 quantised with the all-reduced absmax: the codes the
  // whole-block quantiser gives these features
  const int bn = bitnet_gemm_pick_bn((int)M, (int)H, d.num_sms);
  GemmArgs a{};
  a.M = (int)M; a.N = (int)H; a.K = (int)Ir;
  a.ksplit = plan_ksplit(M, H, Ir, bn, d.num_sms);
  a.scale = s2; a.rowsum = rs2; a.gamma0 = amax2;   // the bf16 rows are not used
  a.y = reinterpret_cast<uint16_t*>(ws + L.yscr);
  a.acc0 = acc;
  if (a.ksplit > 1) {
    a.acc_ws0 = reinterpret_cast<int32_t*>(ws + L.acc0);
    a.tile_cnt = reinterpret_cast<int32_t*>(ws + L.acc0 + splitk_acc_bytes(M, H));
  }
  st = bitnet_quant_launch(h, true, norm2_w, M, Ir, xq2, Ir, true, s2, rs2, nullptr, nullptr, s,
                           amax2, nullptr, a.ksplit > 1 ? ws + L.acc0 : nullptr,
                           a.ksplit > 1 ? splitk_acc_bytes(M, H) + splitk_cnt_bytes(M, H) : 0);
  if (st != BITNET_OK) return st;
  return bitnet_gemm_launch(0 /*linear*/, xq2, down, nullptr, a, bn, d.num_sms, s);
}

bitnet_status bitnet_ffn_tp_finish(const int32_t* acc, int64_t M, int64_t H, int64_t I,
                                   const float* gamma_down, const float* amax2,
                                   const double* sumsq_x, const double* sumsq_h, float eps,
                                   uint16_t* y, float* y_f32, void* stream) {
  if (!acc || !gamma_down || !amax2 || !sumsq_x || !sumsq_h || !y) return BITNET_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || H < 1 || I < 1 || M > 0x7fffffff || H > 0x7fffffff || I > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  if (((uintptr_t)acc & 3u) || ((uintptr_t)y & 1u) || ((uintptr_t)y_f32 & 3u) ||
      ((uintptr_t)amax2 & 3u) || ((uintptr_t)sumsq_x & 7u) || ((uintptr_t)sumsq_h & 7u))
    return BITNET_ERR_ALIGN;
  DevInfo d;
  bitnet_status st = device_info(&d);
  if (st != BITNET_OK) return st;
  int64_t blocks = (M * H + 255) / 256;
  if (blocks > (int64_t)d.num_sms * 8) blocks = (int64_t)d.num_sms * 8;
  ffn_tp_finish_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(
      acc, (int)M, (int)H, (int)I, gamma_down, amax2, sumsq_x, sumsq_h, eps, y, y_f32);
  return cudaGetLastError() == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

bitnet_status bitnet_last_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return BITNET_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return BITNET_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return BITNET_ERR_CUDA;
  }
  return static_cast<bitnet_status>(v);
}

}  // extern "C"
