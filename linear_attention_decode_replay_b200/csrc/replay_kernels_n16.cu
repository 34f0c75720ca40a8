// Replay kernels for k-dim N = 16.
#define REPLAY_N 16
#include "replay_instances.cuh"
