// Single translation unit of the library: the device status word is shared
// by every kernel without relocatable device code.
#include "fa_api.cu"
#include "fa_fwd.cu"
#include "fa_bwd.cu"
#include "fa_quant.cu"
