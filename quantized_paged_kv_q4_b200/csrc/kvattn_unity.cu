// Single translation unit of libkvattn: the per-device error word and every kernel live in
// one module, so no relocatable device code is needed.
#include "quantize.cu"
#include "decode.cu"
#include "merge.cu"
#include "select.cu"
#include "prefill.cu"
#include "stream.cu"
#include "api.cu"
#include "noalloc.cu"
