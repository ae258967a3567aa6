"""B200-native shared-QK LSH attention (Reformer), forward and backward.

The compute lives in ``liblsh.so`` (hand-written sm_100a CUDA kernels behind
the C ABI of ``include/lsh.h``); :mod:`lsh_attention_long_b200.lsh` is its
ctypes binding and :mod:`lsh_attention_long_b200.workloads` draws the seeded
synthetic inputs.
"""

from .lsh import (LshError, Shape, ffn_workspace, forward_host_workspace,  # noqa: F401
                  load_library, lsh_attend_bwd, lsh_attend_fwd, lsh_combine, lsh_device_status,
                  lsh_ffn_backward, lsh_ffn_forward, lsh_forward, lsh_forward_host, lsh_hash, lsh_rev_backward, lsh_rev_forward,
                  lsh_set_wait_test,
                  lsh_sort, lsh_workspace_size, make_shape, rev_workspace, workspace)
