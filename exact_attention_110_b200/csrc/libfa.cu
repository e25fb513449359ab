// Single translation unit for libfa.so: the kernels reference one device status word
// (defined in api.cu), so they are compiled together instead of with relocatable device code.
#include "api.cu"
#include "fa_fwd.cu"
#include "fa_fwd_solo.cu"
#include "fa_fwd_merge.cu"
#include "fa_bwd.cu"
#include "fa_bwd_aux.cu"
#include "fa_bwd_noalloc.cu"
#include "selftest.cu"
