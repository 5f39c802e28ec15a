"""CPU oracle for the DDTree round: test infrastructure only.

Imported by the tests, the package smoke check and the benchmark's CPU
baseline arm; never by the library's compute path.
"""
from .ddtree_oracle import *  # noqa: F401,F403
