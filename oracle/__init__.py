"""Oracle package (TEST INFRASTRUCTURE): plain fp64 CPU statement of the method.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs may import it.  See ``oracle.expert`` (the action expert and
FLASH verification), ``oracle.draft`` (the FLASH draft model and round) and
``oracle.prefill`` (the VLM prefill writing the KV cache) for the cited
passages.
"""

from . import draft, expert, prefill  # noqa: F401
