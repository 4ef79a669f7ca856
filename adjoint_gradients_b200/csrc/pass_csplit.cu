// pass_csplit.cu -- instances of the pass kernel in split form for the fused
// CNOT schedule (two qubit sets, tiles loaded by tensor copies): each pass's
// rotations sit between two diagonal ops and one factor of the layer's CNOT
// map is applied as a permutation of the tile.
#include "pass_kernel.cuh"

#define QML_CSPLIT_INSTANCES(X) X(false, 2, 0, 4) X(true, 2, 0, 4) X(false, 2, 1, 4) X(true, 2, 1, 4)

QML_DEFINE_PASS_UNIT(pass_csplit, QML_CSPLIT_INSTANCES)
