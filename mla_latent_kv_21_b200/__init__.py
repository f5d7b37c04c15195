"""B200-native (sm_100a) MLA decode over a paged latent KV cache.

The compute lives in libmla_decode.so (C ABI, include/mla_decode.h); this
package only marshals arguments to it. Importing the package loads the
library and raises ImportError if it has not been built.
"""

from ._lib import *  # noqa: F401,F403
from ._lib import MlaError, EXPORTED, LIB_PATH  # noqa: F401
from .api import DecodePlan, PrefillPlan, dims_for  # noqa: F401
from .tpla import TplaShardPlan, shard_dims  # noqa: F401
