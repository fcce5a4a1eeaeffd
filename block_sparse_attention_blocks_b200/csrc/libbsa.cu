// Single translation unit of libbsa.so: the kernels share the device error word defined in
// ptx.cuh, so they are compiled together.
#include "pool.cu"
#include "select.cu"
#include "static.cu"
#include "attn.cu"
#include "probe.cu"
#include "capi.cu"
#include "pipeline.cu"
#include "squad.cu"
#include "svg2.cu"
#include "noalloc.cu"
#include "sparsepr.cu"
