// fa_bwd.cuh -- backward pass (to be filled in).
#pragma once
#include "sm100.cuh"
