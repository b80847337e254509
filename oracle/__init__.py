"""CPU oracle (test infrastructure only): see dejavu_oracle.py."""
