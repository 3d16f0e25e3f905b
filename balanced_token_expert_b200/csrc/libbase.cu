// libbase.cu -- the single translation unit of libbase.so (one TU keeps the
// device error word and the kernels in one module without relocatable code).
#include "routing.cu"
#include "auction.cu"
#include "probe.cu"
#include "variant.cu"
#include "gemm.cu"
#include "backward.cu"
#include "ep.cu"
#include "api.cu"
#include "noalloc.cu"
