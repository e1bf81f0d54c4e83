"""CPU oracle (test infrastructure only; never imported by the product path)."""

from .int4_oracle import *  # noqa: F401,F403
from .int4_oracle import __all__ as _sym_all
from .affine_oracle import *  # noqa: F401,F403
from .affine_oracle import __all__ as _affine_all

__all__ = list(_sym_all) + list(_affine_all)
