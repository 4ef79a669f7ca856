// pass_split.cu -- instances of the pass kernel in split form (tangent-form
// Ry rotations and one diagonal op per layer): every fp32 circuit without
// re-uploading or CNOT entanglers.
#include "pass_kernel.cuh"

#define QML_SPLIT_INSTANCES(X)                                                                   \
  X(false, 0, 0, 3) X(true, 0, 0, 3) X(false, 1, 0, 3) X(true, 1, 0, 3) X(false, 1, 1, 3)          \
  X(true, 1, 1, 3) X(false, 2, 0, 3) X(true, 2, 0, 3) X(false, 2, 1, 3) X(true, 2, 1, 3)

QML_DEFINE_PASS_UNIT(pass_split, QML_SPLIT_INSTANCES)
