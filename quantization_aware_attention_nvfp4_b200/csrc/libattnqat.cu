// libattnqat.cu -- the library is compiled as this single translation unit
// (one definition of the device status word, and every kernel template
// instantiated next to its launcher).
#include "quant.cu"
#include "fwd.cu"
#include "bwd.cu"
#include "sparse.cu"
#include "api.cu"
#include "noalloc.cu"
#include "selftest.cu"
