// pass_reup.cu -- instances of the pass kernel with data re-uploading folded
// into the fused SU(2) rotations (form 2: tiles with batch-unit bits, whose
// register pairs span several samples).
#include "pass_kernel.cuh"

#define QML_REUP_INSTANCES(X)                                                                    \
  X(false, 1, 0, 1) X(true, 1, 0, 1) X(false, 1, 1, 1) X(true, 1, 1, 1) X(false, 2, 0, 1)          \
  X(true, 2, 0, 1) X(false, 2, 1, 1) X(true, 2, 1, 1) X(false, 1, 0, 2) X(true, 1, 0, 2)          \
  X(false, 1, 1, 2) X(true, 1, 1, 2)

QML_DEFINE_PASS_UNIT(pass_reup, QML_REUP_INSTANCES)
