// Replay kernels for k-dim N = 128.
#define REPLAY_N 128
#include "replay_instances.cuh"
