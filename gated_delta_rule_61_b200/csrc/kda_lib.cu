// kda_lib.cu -- single translation unit of libkda.so (the device status word
// is shared by every kernel without relocatable device code).
#include "kda_api.cu"
#include "kda_decode.cu"
#include "kda_recurrent.cu"
#include "kda_chunk.cu"
#include "kda_backward.cu"
#include "kda_noalloc.cu"
#include "kda_selftest.cu"
