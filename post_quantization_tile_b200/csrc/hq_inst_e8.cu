// hq_inst_e8.cu -- encode / decode kernels for the E8 lattice.
#include "hq_instantiate.cuh"

HQ_DEFINE_LAUNCHERS(HQ_E8, e8)
