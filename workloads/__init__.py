"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

Holds none of the method's arithmetic: only random draws, a token-grid
positional term, rounding to the input dtype and the per-block redraw of query
noise that keeps routing scores away from near-ties.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    Config,
    config,
    bf16_round,
    generate,
    generate_head,
    redraw_query_block,
    load_redraws,
    small_config,
)
