// Kernels and launchers for head dimension d = 32.
#include "launch_impl.cuh"

SRFTQ_INSTANTIATE_D(32)
