"""sink_augmented_gqa_b200: gpt-oss-style sink-augmented GQA attention on B200.

The product is the C-ABI library ``libsinkattn.so`` (CUDA for sm_100a,
declared in ``include/sinkattn.h``); ``sinkattn`` is its thin ctypes binding
and ``workloads`` holds the seeded synthetic inputs. Importing the package
does not load the library; the first API call does, and raises if it is not
built.
"""

from .sinkattn import (  # noqa: F401
    KVCache,
    SinkAttnError,
    attn_backward,
    attn_decode,
    attn_decode_static,
    attn_prefill,
    decode_workspace,
    decode_workspace_bytes,
    device_status,
    out_proj,
    qkv_proj,
    rmsnorm_fold_weight,
    rope_apply_qk,
    set_prefill_events,
    set_wait_limit,
    yarn_rope_tables,
)
