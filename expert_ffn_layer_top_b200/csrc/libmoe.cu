// Single translation unit of libmoe.so: the device error word and the kernels
// are shared without relocatable device code.
#include "api.cu"
#include "router.cu"
#include "permute.cu"
#include "combine.cu"
#include "ffn_tc.cu"
#include "ffn_mx.cu"
#include "prepack.cu"
#include "cache.cu"
#include "peak.cu"
