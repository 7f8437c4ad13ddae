// libic.cu -- single translation unit of libic_b200.so (one nvcc invocation;
// the kernels share the device error word without relocatable device code).
#include "indexer_tc.cu"
#include "topk.cu"
#include "attn.cu"
#include "misc.cu"
#include "api.cu"
#include "noalloc.cu"
