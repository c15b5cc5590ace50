"""fp64 CPU oracle for MSA (test infrastructure only; never imported by the
product path).  See msa_oracle.py for the definition and its sources."""
from .msa_oracle import *  # noqa: F401,F403
