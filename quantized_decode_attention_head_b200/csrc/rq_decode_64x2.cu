// Decode kernel instantiation for head_dim 64, 2 query heads per kv head.
#include "rq_decode.cuh"

RQ_DECODE_INSTANTIATE(64, 2)
