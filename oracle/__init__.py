"""Float64 CPU oracle of the KronQ layer-quantization path (test infrastructure only)."""
from .kronq import *  # noqa: F401,F403
from .kronq import __all__  # noqa: F401
