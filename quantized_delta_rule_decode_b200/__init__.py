"""B200 (sm_100a) quantised gated Delta-rule decode step (STEPQuant).

A thin Python binding over the C ABI declared in ``include/stepq.h`` and
implemented by the in-tree ``libstepq.so``.  The functions keep the C names
and only marshal arguments (torch tensors -> device pointers, streams -> raw
handles); every step of the decode path runs in the library's CUDA kernels.
There is no fallback: if the library is missing, importing the binding
functions raises.
"""

from ._ffi import (  # noqa: F401
    DTYPE_BF16,
    DTYPE_F32,
    DEV_BAD_SLOT,
    DEV_NONFINITE,
    DEV_TIMEOUT,
    GATE_DIAG,
    GATE_SCALAR,
    MODE_STEPQUANT,
    MODE_UNIFORM,
    TEST_NO_STAGING_COPY,
    UNIT_HEAD,
    UNIT_ROW,
    Plan,
    Pool,
    StepqError,
    library_path,
    load_library,
    stepq_allocate_bits,
    stepq_clear_status,
    stepq_decode_fitpack,
    stepq_decode_readout,
    stepq_decode_step,
    stepq_decode_step_host,
    stepq_decode_step_static,
    stepq_fp32_step,
    stepq_get_status,
    stepq_host_workspace_bytes,
    stepq_impact_weights,
    stepq_lifetime_weight,
    stepq_pack,
    stepq_plan_create,
    stepq_plan_destroy,
    stepq_plan_head_layout,
    stepq_row_impact,
    stepq_unit_distortion,
    stepq_unit_distortion_accumulate,
    stepq_plan_slot_bytes,
    stepq_pool_alloc,
    stepq_pool_free,
    stepq_pool_set_test_faults,
    stepq_unpack,
    stepq_workspace_bytes,
)
