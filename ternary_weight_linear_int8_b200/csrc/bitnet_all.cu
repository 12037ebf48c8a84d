// Single translation unit of the library: the kernels share the device
// status word and helpers without relocatable device code.
#include "common.cuh"
#include "pack.cu"
#include "quant.cu"
#include "gemv.cu"
#include "a48.cu"
#include "resident.cu"
#include "batched.cu"
#include "gemm.cu"
#include "api.cu"
#include "noalloc.cu"
