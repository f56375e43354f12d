// The library as one translation unit: the kernel files share file-scope
// device state (the error word), so they are compiled together.
#include "rope_kv.cu"
#include "decode.cu"
#include "prefill.cu"
#include "gemm.cu"
#include "smallm.cu"
#include "api.cu"
