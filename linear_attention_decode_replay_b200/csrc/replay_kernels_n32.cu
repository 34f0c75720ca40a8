// Replay kernels for k-dim N = 32.
#define REPLAY_N 32
#include "replay_instances.cuh"
