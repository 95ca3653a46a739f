// libftmoe.so is built as a single translation unit: the device status word
// and the kernels share one module, and no relocatable device code is needed.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "ftmoe.h"
#include "sm100.cuh"
#include "profile.cuh"
#include "route.cu"
#include "permute.cu"
#include "combine.cu"
#include "gather.cu"
#include "pack.cu"
#include "ffn.cu"
#include "decode.cu"
#include "selftest.cu"
#include "ffn_host.cu"
#include "layer.cu"
#include "api.cu"
#include "permute_noalloc.cu"
#include "slots.cpp"
#include "ep.cpp"
