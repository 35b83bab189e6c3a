"""fp64 CPU oracle (test infrastructure only; see ``oracle.zebra``)."""
from .zebra import *  # noqa: F401,F403
from .zebra import __all__  # noqa: F401
