"""CPU oracle (test infrastructure only; see nmoe_oracle's header)."""
