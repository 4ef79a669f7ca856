// pass_single.cu -- instances of the pass kernel for the one-launch forward
// of single-tile circuits in split form with one sample per batch unit: the
// amplitude's (re, im) in a lane pair, so twice the tiles of the two-sample
// form, each with half the work.
#include "pass_kernel.cuh"

#define QML_SINGLE_INSTANCES(X) X(false, 1, 0, 5) X(false, 1, 1, 5)

QML_DEFINE_PASS_UNIT(pass_single, QML_SINGLE_INSTANCES)
