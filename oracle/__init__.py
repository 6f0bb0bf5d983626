"""CPU oracle for the DiT denoiser forward — test infrastructure only (see dit_oracle)."""
from . import dit_oracle  # noqa: F401
