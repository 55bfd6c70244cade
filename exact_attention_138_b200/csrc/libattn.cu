// Single translation unit of libattn.so: the C-ABI layer and every kernel are compiled together,
// so the device status word and the shared helpers need no relocatable device code.
#include "api.cu"
#include "fwd_bf16.cu"
#include "fwd_f32.cu"
#include "bwd_bf16.cu"
#include "bwd_noalloc.cu"
#include "ring.cu"
