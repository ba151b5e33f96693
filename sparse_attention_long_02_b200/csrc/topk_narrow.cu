// topk_narrow.cu -- the top-k selection in 256-thread CTAs at <= 64 registers,
// for the chunks of a prefill whose selection runs beside the next chunk's
// indexer (one CTA of each fits on an SM).
#define DSA_TOPK_THREADS 256
#define DSA_TOPK_MIN_CTAS 4
#define DSA_TOPK_LAUNCH launch_topk_narrow
#include "topk_impl.cuh"
