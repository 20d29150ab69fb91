"""CPU oracle for CCA / CCGQA (test infrastructure only; see cca_oracle)."""
from .cca_oracle import *  # noqa: F401,F403
from .cca_oracle import OracleConfig, OracleWeights, OracleState  # noqa: F401
