"""CPU oracle of the GCA paged KV cache (fp64). Test infrastructure only: the product path
never imports it. See gca_oracle.py for the definition and its sources."""
from .gca_oracle import *  # noqa: F401,F403
from .gca_oracle import __all__  # noqa: F401
