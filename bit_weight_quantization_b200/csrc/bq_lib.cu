// Single translation unit of the library: pack, activation and layer kernels
// plus the C ABI (one unit keeps the device error word without relocatable
// device code).
#include "bq_abi.cuh"
