"""Float64 CPU oracle (test infrastructure only; see taylor_oracle.py and oracle.c)."""
