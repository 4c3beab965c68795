"""CPU oracle of the Shannonic INT8 codec — TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm may import this
package. The product path (entropy_coded_lossless_b200) never imports it and shares no code with it.
"""
from .oracle import *  # noqa: F401,F403
