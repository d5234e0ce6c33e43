"""CPU oracle for the GIFT codec (test infrastructure; see gift_oracle.py)."""
