// Single translation unit of libjenga.so: the device error word and wait budget
// are module-global __device__ variables shared by every kernel, so all sources
// are compiled together (no relocatable device code needed).
#include "abi.cu"
#include "movement.cu"
#include "select.cu"
#include "score.cu"
#include "attention.cu"
#include "layer.cu"
#include "lm_loss.cu"
#include "predictor.cu"
#include "score_noalloc.cu"
