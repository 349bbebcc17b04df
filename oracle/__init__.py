"""fp64 CPU oracle for LiteLA.  Test infrastructure: imported only by the tests, the
package smoke check and the benchmark's CPU-baseline leg; never by the product path."""
from .litela_oracle import (  # noqa: F401
    decode_bf16,
    unpack_qkv,
    relu,
    lite_la_rows,
    lite_la_fwd,
    lite_la_block_causal_fwd,
    visible_key_count,
)
from .litela_bwd_oracle import (  # noqa: F401
    lite_la_bwd_head,
    lite_la_bwd,
    lite_la_block_causal_bwd,
)
from .litela_elu_oracle import (  # noqa: F401
    phi_elu1,
    elu1_rows,
    elu1_fwd,
)
from .litela_oproj_oracle import (  # noqa: F401
    linear,
    lite_la_oproj,
)
