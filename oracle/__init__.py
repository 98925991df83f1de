"""CPU fp64 oracle for MLA decode over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the
CUDA path (no kernels, headers, helpers or constants) and it never imports the
``mla_paged_kv_05_b200`` package.
"""

from .mla_oracle import (  # noqa: F401
    D_QK,
    D_V,
    PAGE,
    FP8_PAGE_BYTES,
    decode_bf16,
    decode_e4m3,
    attend_rows,
    gather_latent,
    mla_decode_ref,
    mla_decode_ref_rows,
    unabsorbed_mla,
)
from .cache_append import (  # noqa: F401
    cache_append_ref,
    encode_e4m3,
    quantise_rows_fp8,
)
from .projections import (  # noqa: F401
    absorb_q,
    project_out,
)
from .cascade import (  # noqa: F401
    cascade_decode_ref,
    merge_states,
)
