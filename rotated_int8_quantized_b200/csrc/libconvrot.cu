// libconvrot.cu -- single translation unit of the library (keeps the device
// status word and all kernels in one module without relocatable device code).
#include "rotate_quant.cu"
#include "gemm_i8.cu"
#include "tensor_quant.cu"
#include "api.cu"
#include "noalloc.cu"
