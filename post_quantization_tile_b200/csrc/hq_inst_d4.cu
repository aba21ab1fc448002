// hq_inst_d4.cu -- encode / decode kernels for the D4 lattice.
#include "hq_instantiate.cuh"

HQ_DEFINE_LAUNCHERS(HQ_D4, d4)
