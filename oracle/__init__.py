"""CPU oracle of the QSA decode hot path: test infrastructure only (see qsa_oracle)."""
from .qsa_oracle import *  # noqa: F401,F403
from .qsa_oracle import BLOCK, QsaShape, OracleLayer, PooledKeyCache  # noqa: F401
