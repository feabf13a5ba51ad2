// The whole library as one translation unit. Building it this way (no relocatable device code)
// lets ptxas honour the per-role register budgets (setmaxnreg) of the prefill kernel and inline
// everything across the parts.
#include "attn_api.cu"
#include "attn_fwd.cu"
#include "attn_decode.cu"
#include "attn_decode_static.cu"
#include "attn_fp8.cu"
#include "attn_bwd.cu"
