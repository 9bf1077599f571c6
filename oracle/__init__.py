"""CPU oracle of the QSA layer forward (test infrastructure only; see qsa_oracle.h)."""
