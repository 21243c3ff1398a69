"""CPU oracle of the FlashLoop loop-r attention sublayer.

TEST INFRASTRUCTURE: only the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  It shares no code with the
CUDA library.
"""
from . import flashloop_oracle  # noqa: F401
from .flashloop_oracle import (  # noqa: F401
    QMAX,
    GROUP,
    KVStream,
    OracleDecode,
    OracleSequence,
    PAPER_GROUP,
    PAPER_TAIL,
    PaperKVStream,
    apply_rope,
    cache_bytes,
    dense_causal_attention,
    dense_causal_probs,
    dense_kv_bytes,
    dequantize_groups,
    first_order_storage,
    fixed_mass_update,
    gate,
    gate_norms,
    gate_topk,
    out_projection,
    paper_cache_bytes,
    pack_codes,
    project_qkv,
    quantize_asym,
    dequantize_asym,
    quantize_groups,
    rope_angles,
    sparse_update,
    topk_columns,
    unpack_codes,
)
