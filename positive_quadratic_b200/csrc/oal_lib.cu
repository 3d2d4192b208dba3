// oal_lib.cu -- the whole library as one translation unit, so that device symbols shared by
// all kernels (the error word) exist exactly once without relocatable device code.
#include "oal_common.cuh"
#include "oal_simt.cu"
#include "oal_tc.cu"
#include "oal_api.cu"
#include "oal_host.cu"
#include "oal_hadamard.cu"
#include "oal_varlen.cu"
#include "oal_backward.cu"
#include "oal_backward_chunked.cu"
#include "oal_stateops.cu"
#include "oal_noalloc.cu"
#include "oal_chi.cu"
