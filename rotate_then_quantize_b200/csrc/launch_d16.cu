// Kernels and launchers for head dimension d = 16.
#include "launch_impl.cuh"

SRFTQ_INSTANTIATE_D(16)
