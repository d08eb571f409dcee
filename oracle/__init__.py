"""CPU oracle for the paged KV-cache decode path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and the
two share no code: the only module both sides use is the seeded workload
generator, which holds none of the method's arithmetic.

``pkv_oracle.c`` is the fp64 definition written out (see its header for the
passages it follows); ``brute.py`` is an independent numpy brute force over
contiguous arrays used to pin it.  Every function is pinned by the CPU tests.
"""
from .binding import (  # noqa: F401
    ORACLE_BF16,
    ORACLE_F32,
    blocks_needed,
    build,
    compile_source,
    copy_blocks,
    e4m3_encode,
    e4m3_value,
    gather,
    kv_append,
    kv_append_fp8,
    library_path,
    open_library,
    paged_attention,
    paged_attention_fp8,
    swap_blocks,
    use_library,
    waste_per_sequence,
    waste_physical,
)
