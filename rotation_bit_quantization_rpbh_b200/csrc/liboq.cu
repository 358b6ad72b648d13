// Single translation unit for the device side of liboq, so that the kernels
// and the C ABI share the device error flag without relocatable device code.
#include "rpbh_quant.cu"
#include "rpbh_groups.cu"
#include "rht_big.cu"
#include "qgemm.cu"
#include "api.cu"
