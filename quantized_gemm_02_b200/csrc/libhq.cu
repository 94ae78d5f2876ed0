// Single translation unit for libhq.so: the kernels share the module-scope
// device error word and small inline helpers without relocatable device code.
#include "hq_quant.cu"
#include "hq_pack.cu"
#include "hq_gemm_tc.cu"
#include "hq_gemm_small.cu"
#include "hq_gemm_bs.cu"
#include "hq_moe.cu"
#include "hq_api.cu"
#include "hq_noalloc.cu"
