// moda_lib.cu -- single translation unit of the MoDA library (the kernels and the host
// entry points share the per-device error word, so they are compiled together).
#include "moda_api.cu"
#include "moda_fwd.cu"
#include "moda_bwd.cu"
#include "moda_noalloc.cu"
#include "moda_decode.cu"
#include "moda_kvwrite.cu"
