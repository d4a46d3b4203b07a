// Kernels and launchers for head dimension d = 64.
#include "launch_impl.cuh"

SRFTQ_INSTANTIATE_D(64)
