// Single translation unit for libfa.so.  The kernels share one device-side
// status word and the allocation-free entry point's scratch array; compiling
// them as one unit keeps those symbols local without relocatable device code
// (which would also stop ptxas from honouring per-warpgroup register budgets).
#include "fa_api.cu"
#include "fa_simt.cu"
#include "fa_fwd_sm100.cu"
#include "fa_bwd_sm100.cu"
