// Single translation unit for the whole library: the kernels share the
// library's device-side error word and wait cap without relocatable device code.
#include <string.h>
#include "permute.cu"
#include "exchange.cu"
#include "attn_fwd_sm100.cu"
#include "attn_bwd_sm100.cu"
#include "proj_sm100.cu"
#include "api.cu"
#include "bwd_noalloc.cu"
#include "host_pipeline.cu"
