// decode step (to come)
#include "sm100.cuh"
