"""CPU oracle (test infrastructure only; see kq_oracle.h)."""
