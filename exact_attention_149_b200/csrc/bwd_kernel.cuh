// Backward attention kernels (filled in below the forward path).
#pragma once
#include "ptx.cuh"
