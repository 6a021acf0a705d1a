// libsp24 is built as one translation unit so that the per-device status word
// and the helpers are shared without relocatable device code.
#include "api.cu"
#include "prune.cu"
#include "gemm_sp.cu"
#include "permute.cu"
#include "conv.cu"
