// moe_lib.cu -- single translation unit of the library (one device error word
// shared by every kernel without relocatable device code).
#include "api.cu"
#include "balance.cu"
#include "capacity.cu"
#include "capacity_static.cu"
#include "dispatch_combine.cu"
#include "ffn.cu"
#include "ffn_simt.cu"
#include "ffn_tc.cu"
#include "ffn_fused.cu"
#include "router.cu"
#include "router_tc.cu"
#include "stats.cu"
