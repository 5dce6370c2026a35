// Single translation unit of librbd.so: the device status word defined in
// rbd_api.cu is referenced by kernels of the other files, so they are compiled
// together (no relocatable device code needed).
#include "rbd_api.cu"
#include "rbd_prologue.cu"
#include "rbd_gemm.cu"
#include "rbd_skinny.cu"
#include "rbd_nvfp4.cu"
#include "rbd_kv4.cu"
#include "rbd_rope.cu"
#include "rbd_attn.cu"
#include "rbd_svdquant.cu"
