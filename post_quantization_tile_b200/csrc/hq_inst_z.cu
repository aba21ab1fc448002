// hq_inst_z.cu -- encode / decode kernels for the Z lattice.
#include "hq_instantiate.cuh"

HQ_DEFINE_LAUNCHERS(HQ_Z, z)
