"""B200-native edge-conditioned E(3)-equivariant tensor-product convolution.

The computation lives in libtp.so (CUDA C++ for sm_100a, C ABI in include/tp.h).  This
package only loads it and marshals torch tensors into its calls.  There is no other path:
the first call (plan creation, any op, load()) raises ImportError when the library has not
been built.  Importing the package itself does not need the library, so that its build
module (`python -m equivariant_tensor_product_b200.build`) runs in a fresh checkout.
"""
from ._lib import (TP_FLAG_CHECK_INDICES, TP_LINEAR_CUDA_CORES, TP_LINEAR_TENSOR_CORES, TP_MODE_UVU, TP_MODE_UVW, TP_OP_BWD, TP_OP_DBWD, TP_OP_FWD,  # noqa: F401
                   TPError, load)
from .ops import (Plan, tp_conv_bwd, tp_conv_dbwd, tp_conv_fwd, tp_csr_transpose, tp_csr_transpose_workspace_size,  # noqa: F401
                  tp_conv_bwd_radial, tp_conv_fwd_radial, tp_get_device_error, tp_radial_workspace_size,
                  tp_plan_create, tp_plan_query, tp_version, tp_workspace_size)
from .autograd import GateFn, LinearFn, TPConv, TPConvRadial, tp_conv, tp_conv_radial, tp_gate, tp_linear  # noqa: F401
from .block import (Gate, Linear, tp_gate_bwd, tp_gate_dbwd, tp_gate_fwd, tp_linear_bwd, tp_linear_fwd,  # noqa: F401
                    tp_linear_workspace_size)
from .gaunt import Gaunt, tp_gaunt_bwd, tp_gaunt_fwd, tp_gaunt_workspace_size  # noqa: F401
