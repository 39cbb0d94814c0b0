// Single translation unit for the device code of libpa: the kernels share one
// device error word, so they are compiled together (no relocatable device code).
#include "pa_decode.cu"
#include "pa_cache.cu"
#include "pa_extend.cu"
#include "pa_extend_tc.cu"
