// Single translation unit of libmoeq (the device error word and wait budget
// are plain __device__ globals shared by every kernel, without relocatable
// device code).
#include "api.cu"
#include "adapter.cu"
#include "combine.cu"
#include "ep.cu"
#include "gemm.cu"
#include "route.cu"
