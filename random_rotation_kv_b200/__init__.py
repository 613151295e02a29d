"""random_rotation_kv_b200 — random-rotation KV / embedding vector quantisation on B200.

The hot path lives in ``librrq.so`` (hand-written sm_100a CUDA kernels behind the
C ABI declared in ``include/rrq.h``).  This package holds:

* ``binding``   — ctypes binding with the C names (``rrq_encode``, ``rrq_decode``,
                  ``rrq_qk_scores``, ``rrq_q4_0_rot``, ...) on torch CUDA tensors;
* ``build``     — builds ``librrq.so`` in-tree for sm_100a;
* ``workloads`` — seeded synthetic inputs for the five workloads.

The library is loaded on first use; calls fail loudly if it is missing.
"""

from .binding import (  # noqa: F401
    DTYPE_CODE,
    LIB_PATH,
    RRQError,
    lib,
    rrq_attention_decode,
    rrq_attention_workspace_bytes,
    rrq_codebook,
    rrq_decode,
    rrq_drive_encode,
    rrq_encode,
    rrq_format_version,
    rrq_ggml_block_bytes,
    rrq_ggml_rot,
    rrq_ggml_rot_decode,
    rrq_q4_0_rot,
    rrq_q4_0_rot_decode,
    rrq_qjl_matrix,
    rrq_qk_scores,
    rrq_qk_scores_qjl,
    rrq_rotate,
    strerror,
)
