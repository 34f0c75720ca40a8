// Replay kernels for k-dim N = 64.
#define REPLAY_N 64
#include "replay_instances.cuh"
