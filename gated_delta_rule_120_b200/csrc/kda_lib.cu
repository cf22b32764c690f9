// kda_lib.cu — single translation unit of libkda.so. The kernel files share one per-device
// status word (defined in kda_common.cuh), so they are compiled together rather than linked with
// relocatable device code.
#include "kda_api.cu"
#include "kda_profile.cu"
#include "kda_recurrent_chunk.cu"
#include "kda_decode.cu"
#include "kda_chunk_simt.cu"
#include "kda_chunk_tc.cu"
#include "kda_epilogue.cu"
#include "kda_chunk_bwd.cu"
#include "kda_noalloc.cu"
#include "kda_selftest.cu"
