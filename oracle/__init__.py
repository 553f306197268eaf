"""CPU oracle of the ALoDLM denoising step (test infrastructure; see alodlm_oracle)."""
from .alodlm_oracle import Oracle, RULE_PAPER, RULE_PER_TOKEN  # noqa: F401
