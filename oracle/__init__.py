"""HiLS CPU oracle (test infrastructure only; see oracle.py and hils_oracle.c)."""
