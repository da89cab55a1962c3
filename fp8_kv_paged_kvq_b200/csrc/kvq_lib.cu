// Single translation unit of libkvq.so: the kernels share one device-side
// error word, so they are compiled together.
#include "append.cu"
#include "validate.cu"
#include "decode_gqa.cu"
#include "decode_wide.cu"
#include "api.cu"
#include "decode_noalloc.cu"
