// Kernels and launchers for head dimension d = 128.
#include "launch_impl.cuh"

SRFTQ_INSTANTIATE_D(128)
