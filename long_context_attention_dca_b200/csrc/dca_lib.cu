// Single translation unit of the library: every kernel file is included here
// so that the device error word in dca_api.cu is one object shared by all
// kernels without relocatable device code.
#include "dca_api.cu"
#include "rope.cu"
#include "index_map.cu"
#include "attn_prefill_mma.cu"
#include "attn_prefill_sm100_pp.cu"
#include "attn_prefill_sm100_gen.cu"
#include "attn_decode.cu"
#include "decode_noalloc.cu"
#include "prefill_host.cu"
