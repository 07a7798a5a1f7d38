"""Float64 CPU oracle for content-routed block-sparse attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path.  It shares
no code with the CUDA library.  Every function cites the passage it follows;
``reference.py`` holds the implementation and lists the reading taken at
every point the pages leave open.
"""
from .reference import *  # noqa: F401,F403
from .reference import __all__  # noqa: F401
