"""CPU oracle of the GSA layer (test infrastructure only; see gsa_oracle.py)."""
from .gsa_oracle import *  # noqa: F401,F403
from .flashvggt_oracle import bilinear_resize, descriptor_attention_head, descriptors, resize_weights  # noqa: F401
from . import gsa_backward_oracle  # noqa: F401
