// Single translation unit of libwkv7.so: the sticky device status word is one
// __device__ variable shared by every kernel, so all kernels are compiled
// together (no relocatable device code needed).
#include "wkv7_api.cu"
#include "fwd_seq.cu"
#include "step.cu"
#include "bwd_chunk.cu"
#include "bwd_chunk_tc.cu"
#include "bwd_dchain.cu"
#include "fwd_chunk.cu"
#include "bwd_noalloc.cu"
#include "fwd_host.cu"
#include "timemix.cu"
