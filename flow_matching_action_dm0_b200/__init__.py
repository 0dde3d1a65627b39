"""B200-native flow-matching action-expert suffix loop with FLASH verification.

The computation lives in ``librtv.so`` (CUDA, sm_100a; C ABI in
``include/rtv.h``).  This package holds the ctypes binding (``_lib``), a
small handle class (``expert.ActionExpert``), the FLASH draft model and
round (``draft.DraftModel``, ``draft.flash_round``), the VLM prefill that
writes the expert's cache (``prefill.PrefillStack``), the build script
(``build``) and the replica plumbing for several GPUs (``replicas``).
"""

from . import _lib  # noqa: F401
from ._lib import RtvError, load_library  # noqa: F401
from .draft import DraftModel, flash_round, make_draft_config  # noqa: F401
from .expert import ActionExpert, make_config  # noqa: F401
from .prefill import PrefillStack, make_prefill_config  # noqa: F401
