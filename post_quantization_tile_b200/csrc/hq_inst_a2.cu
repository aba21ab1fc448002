// hq_inst_a2.cu -- encode / decode kernels for the A2 lattice.
#include "hq_instantiate.cuh"

HQ_DEFINE_LAUNCHERS(HQ_A2, a2)
