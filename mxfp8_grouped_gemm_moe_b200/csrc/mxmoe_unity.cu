// Single translation unit for libmxmoe.so (the device status word is shared by all
// kernels without relocatable device code).
#include "route.cu"
#include "route_noalloc.cu"
#include "router.cu"
#include "quantize.cu"
#include "gemm.cu"
#include "api.cu"
#include "api_bf16.cu"
