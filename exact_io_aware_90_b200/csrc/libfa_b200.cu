// libfa_b200.cu — single translation unit of libfa_b200.so: the kernels and
// the C ABI share the device status word without relocatable device code.
#include "fa_api.cu"
#include "fa_fwd.cu"
#include "fa_bwd.cu"
#include "fa_decode.cu"
#include "fa_merge.cu"
#include "fa_noalloc.cu"
